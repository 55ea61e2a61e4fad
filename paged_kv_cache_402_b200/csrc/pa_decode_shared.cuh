// Cascade decode over shared prefix blocks (bf16, head_dim 128, group size
// 1..8, tensor cores): the partitions that several sequences of a batch hold
// in the same physical blocks are read once for all of them.
//
// The pages make sharing the point of the paged layout: sequences with a
// common prefix, or the samples of one request, point at the same physical
// blocks ("pagedattention" glossary entry, comparison table and paragraph 5;
// "PagedAttention Internals", "Sharing And Dynamic Growth").  The attention
// of each sequence over such a block is still its own: this kernel computes,
// for a group of up to kSlots sequences whose block tables agree on their
// first `shared` tokens (a whole number of blocks), each member's
// split-context statistics (max, sum, unnormalised accumulator) of those
// tokens, cut at the partition boundaries: the whole partitions among them
// go to the rows decode_partition_tc would write for them, the piece of the
// partition the shared tokens end in (if they end inside one) to the
// member's extra row.  decode_partition_tc then does every sequence from its
// first private token on, and the log-sum-exp reduce merges them all.
//
// Same machinery as decode_partition_tc (see there): persistent CTAs, a TMA
// producer warp loading whole (block, kv head) tiles as 4-D boxes into
// 128-byte-swizzled K and V rings, softmax warps with the lazy reference and
// the transposed column reductions.  What differs:
//  * two MMA lanes: warp 1 issues the QKs, warp 10 the PVs (one lane issuing
//    both streams in order set the pace: a chunk's PV waited behind the next
//    chunk's K tile and QK issue);
//  * a work unit is (group, kv head, piece): a whole partition or the
//    shorter piece at the end of the shared tokens, handed out round-robin;
//    the producer loads the next unit's description while the current
//    unit's copies are in flight;
//  * the Q tile holds the group's members in 8-row slots (member m: rows
//    8m .. 8m + G - 1, one 2-D TMA box per column half per member), so the
//    MMAs are M = 128 tokens x N = 32 query rows;
//  * two softmax warpgroups (warps 2-5 and 6-9) take columns 0-15 and 16-31
//    of S and O, each with its own running statistics and named barrier;
//  * the epilogue writes workspace rows for every (member, query head), read
//    from O at the start of the next unit (the PV lane issues a unit's last
//    PV as soon as its P is in, so it does not wait for the next unit's
//    first K tile);
//  * two K and three V ring slots (the larger Q and P tiles take the third K
//    slot's room; a V tile is held longer, until its PV has run).
#pragma once

#include "pa_decode_tc.cuh"

namespace pa {

struct ShLayout {
  static constexpr int kSlots = 4;          // sequences per unit
  static constexpr int kN = 8 * kSlots;     // MMA N: 8 query rows per member slot
  static constexpr int kChunk = 128;
  // ring slots: a V tile is held until its chunk's PV has run (after the
  // softmax), a K tile only until its QK has, so V gets the third slot
  static constexpr int kKStages = 2;
  static constexpr int kVStages = 3;
  static constexpr int kTile = kChunk * 256;
  static constexpr int kGroup = 2048;
  static constexpr int kQ = 2 * kN * 128;   // two column halves of kN rows x 128 B
  static constexpr int kP = 2 * kN * 128;   // two 64-token halves of kN rows x 128 B
  static constexpr int kMaxGroups = 1024;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKStages * kTile;
  static constexpr int kOffQ = kOffV + kVStages * kTile;
  static constexpr int kOffP = kOffQ + 2 * kQ;
  static constexpr int kOffBar = kOffP + 2 * kP;
  static constexpr int kNumBars = 23;
  static constexpr int kOffRed = kOffBar + (kNumBars * 8 + 15) / 16 * 16;  // 16-byte aligned
  static constexpr int kRedFloats = 2 * 4 * kN;  // [parity][warp][column]
  static constexpr int kOffRedSum = kOffRed + kRedFloats * 4;
  static constexpr int kOffTmem = kOffRedSum + kRedFloats * 4;
  // unit slot: [group, kv head, workspace row, members, b_0 .. b_3, chunks,
  // -, -, -] + the table entries of the piece (from the first member's table)
  static constexpr int kUnitHead = 12;
  static constexpr int kUnitInts = kUnitHead + TcLayout::kMaxPart / 8;
  static constexpr int kOffUnit = kOffTmem + 16;
  static constexpr int kOffScan = kOffUnit + 2 * kUnitInts * 4;
  static constexpr int kOffPrefix = kOffScan + 64;  // pieces before each group
  static constexpr int kOffShared = kOffPrefix + (kMaxGroups + 1) * 4;  // each group's shared tokens
  static constexpr int kBytes = kOffShared + kMaxGroups * 4 + 1024;
  static constexpr int kThreads = 352;  // producer, QK lane, 8 softmax warps, PV lane
  static constexpr uint32_t kTmemCols = 128;  // S0 S1 O0 O1, kN columns each
};

static_assert(ShLayout::kBytes <= 227 * 1024, "shared memory of the cascade kernel");

// OR of `pred` over the 128 threads of softmax warpgroup `grp` (named
// barrier 1 + grp).
__device__ __forceinline__ bool grp_sync_or(int pred, int grp) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(1 + grp)
      : "memory");
  return r != 0;
}

// The sharing plan of one launch: group j has members[j * max_members + m]
// (m < max_members, -1 past its last member) sharing their first shared[j]
// tokens (a whole number of blocks).
struct SharedParams {
  const int32_t *members;
  const int32_t *shared;
  int32_t n_groups;
  int32_t max_members;
};

// One CTA of 352 threads per SM.  Each of the SM's four sub-partitions
// holds 16 K registers and three of the eleven warps land on three of them,
// so a thread gets at most 168.
// PART: tokens per partition (256, 512 or 1024); the caller's p.part.
template <int G, int PART>
__global__ void __launch_bounds__(ShLayout::kThreads, 1)
    decode_shared_tc(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v,
                     const __grid_constant__ CUtensorMap tmap_q, DecodeParams p, SharedParams sp) {
  using L = ShLayout;
  constexpr int N = L::kN;
  static_assert(G >= 1 && G <= 8, "group size");
  static_assert(PART == 256 || PART == 512 || PART == 1024, "partition size");
  constexpr int NE = PART / 8 / 32;  // table entries per lane of a unit (bs >= 8)
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *kfull = bars, *kempty = bars + 2, *vfull = bars + 4, *vempty = bars + 7;
  uint64_t *qfull = bars + 10, *qempty = bars + 12, *sfull = bars + 14, *pfull = bars + 16;
  uint64_t *pvdone = bars + 18, *ofree = bars + 20, *drain = bars + 22;
  int32_t *gprefix = reinterpret_cast<int32_t *>(smem + L::kOffPrefix);
  int32_t *gshared = reinterpret_cast<int32_t *>(smem + L::kOffShared);
  int32_t *scan = reinterpret_cast<int32_t *>(smem + L::kOffScan);
  int32_t *unit_slots = reinterpret_cast<int32_t *>(smem + L::kOffUnit);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmem);
  float *red_max = reinterpret_cast<float *>(smem + L::kOffRed);
  float *red_sum = reinterpret_cast<float *>(smem + L::kOffRedSum);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kKStages; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < L::kVStages; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 4);  // the QK lane's commit, each softmax warpgroup, the PV lane
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 256);
      mbar_init(&pvdone[i], 1);
      mbar_init(&ofree[i], 256);
    }
    mbar_init(drain, 2);  // the QK and the PV lanes' last commits
    fence_barrier_init();
  }
  // Q rows a member slot does not use (G..7) and unused P rows stay zero
  for (int i = threadIdx.x; i < (2 * L::kQ + 2 * L::kP) / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(smem + L::kOffQ)[i] = make_uint4(0, 0, 0, 0);

  // pieces per group (its shared tokens cut at the partition boundaries) and
  // their exclusive prefix sums (the plan is caller data that no kernel of
  // the library writes: read before the wait)
  const int NG = sp.n_groups;
  constexpr int kMaxSeg = (L::kMaxGroups + L::kThreads - 1) / L::kThreads;
  const int seg = (NG + blockDim.x - 1) / blockDim.x;
  const int j_first = threadIdx.x * seg;
  int cnt[kMaxSeg];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < kMaxSeg; ++i) {
    cnt[i] = 0;
    const int j = j_first + i;
    if (i < seg && j < NG) {
      const int S = sp.shared[j];
      if (S < 0 || S % p.bs != 0 || S / p.bs > p.max_blocks) {
        if (blockIdx.x == 0) raise_error(PA_DEVERR_PLAN);
      } else {
        cnt[i] = (S + PART - 1) / PART;
      }
      gshared[j] = S;
      mine += cnt[i];
    }
  }
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  if (warp == 1) tc::tmem_alloc(tmem_slot, L::kTmemCols);
  __syncthreads();
  int run = incl - mine;
  for (int w = 0; w < warp; ++w) run += scan[w];
#pragma unroll
  for (int i = 0; i < kMaxSeg; ++i) {
    const int j = j_first + i;
    if (i < seg && j < NG) {
      gprefix[j] = run;
      run += cnt[i];
      if (j == NG - 1) gprefix[NG] = run;
    }
  }
  if (warp == 1) tc::tmem_relinquish();
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int num_units = p.Hkv * gprefix[NG];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tensormap(&tmap_k);
      tc::prefetch_tensormap(&tmap_v);
      tc::prefetch_tensormap(&tmap_q);
    }
    const uint64_t pol_kv = policy_evict_first();
    const uint64_t pol_q = tc::policy_evict_last();
    const int bs = p.bs;
    const int blocks_per_chunk = L::kChunk / bs;
    const int oob_group = p.num_blocks * p.Hkv * (bs / 8);
    const int lg_bs = bs == 8 ? 3 : (bs == 16 ? 4 : 5);
    int c = 0, qi = 0;
    bool ok = true;
    // unit u: kv head u % Hkv of piece u / Hkv in the groups' order
    struct ShUnit {
      int j, g, row, nmem, nb, nchunks;
      int32_t b[L::kSlots];
    };
    auto pick = [](const int32_t (&x)[NE], int k) {  // x[k] by selects, never a local-memory index
      int32_t v = x[0];
#pragma unroll
      for (int i = 1; i < NE; ++i) v = select_i32(k == i, x[i], v);
      return v;
    };
    auto load_unit = [&](int u, ShUnit &un, int32_t (&x)[NE]) {
#pragma unroll
      for (int k = 0; k < NE; ++k) x[k] = -1;
      un.nmem = 0;
      if (u >= num_units) return;
      const int w = u / p.Hkv;
      un.g = u - w * p.Hkv;
      int lo = 0, hi = NG - 1;  // largest group whose count before it is <= w
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (gprefix[mid] <= w) lo = mid; else hi = mid - 1;
      }
      un.j = lo;
      // piece k: tokens [k PART, min((k + 1) PART, S)); a whole partition
      // goes to row k, the shorter last piece to the extra row max_parts
      const int k = w - gprefix[lo], S = gshared[lo];
      const int t0 = k * PART, t1 = min(t0 + PART, S);
      un.row = t1 - t0 == PART ? k : p.max_parts;
      un.nb = (t1 - t0) >> lg_bs;
      un.nchunks = (t1 - t0 + L::kChunk - 1) / L::kChunk;
      const int32_t mb = lane < L::kSlots && lane < sp.max_members ? sp.members[(size_t)lo * sp.max_members + lane] : -1;
      int nmem = 0;
#pragma unroll
      for (int m = 0; m < L::kSlots; ++m) {
        un.b[m] = __shfl_sync(0xffffffffu, mb, m);
        if (un.b[m] >= 0 && un.b[m] < p.B && nmem == m) nmem = m + 1;
      }
      un.nmem = nmem;
      if (nmem == 0) return;
      const int32_t *tr = p.tables + (size_t)un.b[0] * p.max_blocks + (t0 >> lg_bs);
#pragma unroll
      for (int e = 0; e < NE; ++e)
        if (lane + 32 * e < un.nb) x[e] = tr[lane + 32 * e];
    };
    ShUnit un{}, nx{};
    int32_t e[NE], f[NE];
    int u = blockIdx.x;
    load_unit(u, un, e);
    wait_prior_grid();  // the copies read the pool and Q, which may be written just before
    allow_next_grid();
    while (ok && u < num_units) {
      // The next unit's description (members, table entries) is loaded while
      // this unit's copies are in flight: after its second chunk's loads,
      // where the two-stage ring makes the producer wait anyway.
      bool have_next = false;
      if (un.nmem > 0) {
        const int qs = qi & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&qempty[qs], ((qi >> 1) & 1) ^ 1))) { ok = false; break; }
        {
          int32_t *us = unit_slots + qs * L::kUnitInts;
          if (lane == 0) {
            us[0] = un.j;
            us[1] = un.g;
            us[2] = un.row;
            us[3] = un.nmem;
#pragma unroll
            for (int m = 0; m < L::kSlots; ++m) us[4 + m] = un.b[m];
            us[8] = un.nchunks;
          }
#pragma unroll
          for (int k = 0; k < NE; ++k) us[L::kUnitHead + 32 * k + lane] = e[k];
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&qfull[qs], un.nmem * 2 * G * 128);
          uint8_t *qdst = smem + L::kOffQ + qs * L::kQ;
          for (int m = 0; m < un.nmem; ++m) {
            const int qy = un.b[m] * p.Hq + un.g * G;
            tc::tma_load_2d(qdst + m * 8 * 128, &tmap_q, 0, qy, &qfull[qs], pol_q);
            tc::tma_load_2d(qdst + N * 128 + m * 8 * 128, &tmap_q, 64, qy, &qfull[qs], pol_q);
          }
        }
        ++qi;
        for (int ci = 0; ci < un.nchunks; ++ci, ++c) {
          for (int which = 0; which < 2; ++which) {  // 0: K ring, 1: V ring
            const int st = which ? L::kVStages : L::kKStages;
            const int slot = c % st, use = c / st;
            uint64_t *empty = which ? &vempty[slot] : &kempty[slot];
            uint64_t *full = which ? &vfull[slot] : &kfull[slot];
            const CUtensorMap *map = which ? &tmap_v : &tmap_k;
            if (!__all_sync(0xffffffffu, mbar_wait(empty, (use & 1) ^ 1))) { ok = false; break; }
            uint8_t *dst = smem + (which ? L::kOffV : L::kOffK) + slot * L::kTile;
            if (lane == 0) mbar_arrive_expect_tx(full, L::kTile);
            __syncwarp();
            const int jloc = ci * blocks_per_chunk + (lane % blocks_per_chunk);
            const int32_t blk = __shfl_sync(0xffffffffu, pick(e, (ci * blocks_per_chunk) >> 5), jloc & 31);
            if (lane < blocks_per_chunk) {
              int w = oob_group;  // past the piece's last block: the fill value
              if (jloc < un.nb) {
                if (blk >= 0 && blk < p.num_blocks) w = (blk * p.Hkv + un.g) * (bs / 8);
                else if (which == 0) raise_error(PA_DEVERR_TABLE);
              }
              tc::tma_load_4d(dst + lane * (bs / 8) * L::kGroup, map, 0, 0, 0, w, full, pol_kv);
            }
          }
          if (!ok) break;
          if (ci == 1) {
            load_unit(u + gridDim.x, nx, f);
            have_next = true;
          }
        }
        if (!ok) break;
      }
      if (!have_next) load_unit(u + gridDim.x, nx, f);
      u += gridDim.x;
      un = nx;
#pragma unroll
      for (int k = 0; k < NE; ++k) e[k] = f[k];
    }
    if (ok) {  // no work left: an empty unit stops the consumers
      const int qs = qi & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&qempty[qs], ((qi >> 1) & 1) ^ 1))) {
        ok = false;
      } else {
        if (lane == 0) unit_slots[qs * L::kUnitInts + 3] = 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfull[qs]);
      }
    }
    if (!ok && lane == 0) {
      raise_error(PA_DEVERR_TIMEOUT);
      for (int k = (c > L::kVStages ? c - L::kVStages : 0); k <= c; ++k) {
        mbar_wait(&kfull[k % L::kKStages], (k / L::kKStages) & 1, 100000000ull);
        mbar_wait(&vfull[k % L::kVStages], (k / L::kVStages) & 1, 100000000ull);
      }
      for (int k = (qi > 2 ? qi - 2 : 0); k < qi; ++k) mbar_wait(&qfull[k & 1], (k >> 1) & 1, 100000000ull);
    }
  } else if (warp == 1 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // Two lanes issue the MMAs, so that neither waits behind the other's
    // stream: warp 1 the QKs (as each K tile lands, and once the softmax has
    // written P(c - 2), so has read S(c - 2) whose buffer QK(c) takes), warp
    // 10 the PVs (as each chunk's P and V are in).  Each commits its own
    // barriers; the softmax waits for PV(c - 2) before it writes P(c) over
    // P(c - 2)'s buffer.
    wait_prior_grid();
    allow_next_grid();
    constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(128, N, false, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(128, N, true, false);
    const uint32_t kbase0 = smem_u32(smem + L::kOffK), vbase0 = smem_u32(smem + L::kOffV);
    const uint32_t qbase0 = smem_u32(smem + L::kOffQ), pbase0 = smem_u32(smem + L::kOffP);
    const bool qk_lane = warp == 1;
    bool ok = true;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    int c = 0, qi = 0;
    while (ok) {
      const int qs = qi & 1;
      if (!warp_wait(&qfull[qs], (qi >> 1) & 1)) { ok = false; break; }
      const int nmem = unit_slots[qs * L::kUnitInts + 3];
      const uint32_t qb = qbase0 + qs * L::kQ;
      const int nchunks = unit_slots[qs * L::kUnitInts + 8];
      if (!qk_lane) {  // the PV lane has read the unit: the slot may be taken again
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qs]);
      }
      if (nmem == 0) break;  // the producer ran out of work
      for (int ci = 0; ci < nchunks; ++ci, ++c) {
        const int slot = c % L::kKStages, vslot = c % L::kVStages;
        if (qk_lane) {
          if (!warp_wait(&kfull[slot], (c / L::kKStages) & 1)) { ok = false; break; }
          if (c >= 2 && !warp_wait(&pfull[c & 1], ((c - 2) >> 1) & 1)) { ok = false; break; }
          if (lane == 0) {
            tc::fence_after_sync();
            const uint32_t kb = kbase0 + slot * L::kTile;
            const uint32_t d = tmem + (c & 1) * N;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * 1024 + (kk & 3) * 32;
              const uint64_t a = tc::smem_desc_sw128(kb + koff, 16, L::kGroup);
              const uint64_t bdesc = tc::smem_desc_sw128(qb + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
              tc::mma_bf16(d, a, bdesc, idesc_qk, kk > 0);
            }
            tc::mma_commit(&sfull[c & 1]);
            tc::mma_commit(&kempty[slot]);
            if (ci == nchunks - 1) tc::mma_commit(&qempty[qs]);
          }
          __syncwarp();
        } else {
          if (!warp_wait(&pfull[c & 1], (c >> 1) & 1)) { ok = false; break; }
          if (!warp_wait(&vfull[vslot], (c / L::kVStages) & 1)) { ok = false; break; }
          // the accumulator is free once the epilogue of the unit two back read it
          if (ci == 0 && !warp_wait(&ofree[qi & 1], ((qi >> 1) & 1) ^ 1)) { ok = false; break; }
          if (lane == 0) {
            tc::fence_after_sync();
            const uint32_t vb = vbase0 + vslot * L::kTile;
            const uint32_t pb = pbase0 + (c & 1) * L::kP;
            const uint32_t d = tmem + 2 * N + (qi & 1) * N;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t a = tc::smem_desc_sw128(vb + kk * 2 * L::kGroup, 1024, L::kGroup);
              const uint64_t bdesc = tc::smem_desc_sw128(pb + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
              tc::mma_bf16(d, a, bdesc, idesc_pv, (kk > 0 || ci > 0) ? 1u : 0u);
            }
            tc::mma_commit(&pvdone[c & 1]);
            tc::mma_commit(&vempty[vslot]);
          }
          __syncwarp();
        }
      }
      ++qi;
    }
    if (!ok && lane == 0) raise_error(PA_DEVERR_TIMEOUT);
    // no MMA of this lane may still be running when the CTA frees its tensor memory
    if (lane == 0) tc::mma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Two warpgroups split the columns: warps 2-5 take columns 0-15 of S and
    // O (member slots 0 and 1), warps 6-9 columns 16-31 (slots 2 and 3).
    // Columns are independent, so each group keeps its own running maxima
    // and sums, lazy reference and reductions (named barrier 1 + group).
    wait_prior_grid();  // before the first write of the workspace
    allow_next_grid();
    constexpr int NC = N / 2;         // columns of one warpgroup
    const int grp = (warp - 2) >> 2;  // 0: warps 2-5, 1: warps 6-9
    const int c0 = grp * NC;          // the group's first column
    const int wq = warp & 3;          // the warp's quarter of the TMEM lanes
    const int r = wq * 32 + lane;     // token row (softmax) / head-dim row (O)
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const int bs = p.bs;
    const int log2_bs = bs == 8 ? 3 : (bs == 16 ? 4 : 5);
    float m[NC], l[NC];
    int pun_g = 0, pun_row = 0, pun_nmem = 0, pun_b[L::kSlots] = {0, 0, 0, 0};
    bool pend = false;
    int p_clast = 0, p_u = 0;
    bool bad = false, stop = false;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      if (!bad && !__all_sync(0xffffffffu, mbar_wait(bar, parity))) bad = true;
    };
    // column n of S / O: member slot n / 8, query head n % 8 of the group
    auto col_valid = [&](int n, int nmem) { return (n >> 3) < nmem && (n & 7) < G; };
    // [group][parity][warp][column] partial maxima and sums
    auto red_at = [&](float *base, int parity) { return base + (grp * 2 + parity) * 4 * NC; };

    // the previous unit's O and sums -> its members' workspace rows
    auto epilogue = [&]() {
      float o[NC];
      warp_wait(&pvdone[p_clast & 1], (p_clast >> 1) & 1);
      if (!bad) {
        tc::fence_after_sync();
        tc::tmem_ld16(trow + 2 * N + (p_u & 1) * N + c0, o);
      }
      tc::fence_before_sync();
      mbar_arrive(&ofree[p_u & 1]);
      float *rs = red_at(red_sum, p_u & 1);
      {  // this warp's part of every column's sum; lane j (and j + 16) holds column j
        float v[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j) v[j] = l[j];
        const float t = warp_reduce_columns<NC, false>(v, lane);
        if (lane < NC) rs[wq * NC + lane] = t;
      }
      stop = grp_sync_or(bad, grp);
      if (stop) return;
      // workspace rows of the group's two member slots at query head 0;
      // column j is row rb[j / 8] + (j % 8) * row_stride
      const size_t hb = (size_t)pun_g * G;
      const size_t rb0 = ((size_t)(grp ? pun_b[2] : pun_b[0]) * p.Hq + hb) * p.row_stride + pun_row;
      const size_t rb1 = ((size_t)(grp ? pun_b[3] : pun_b[1]) * p.Hq + hb) * p.row_stride + pun_row;
      auto ws_row = [&](int j) { return (j < 8 ? rb0 : rb1) + (size_t)(j & 7) * p.row_stride; };
#pragma unroll
      for (int j = 0; j < NC; ++j)
        if (col_valid(c0 + j, pun_nmem)) p.ws_acc[ws_row(j) * 128 + r] = o[j];
      if (wq == 0 && lane < NC && col_valid(c0 + lane, pun_nmem)) {  // lane j: column j's max and sum
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) Ls += rs[w * NC + lane];
        float mj = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j)
          if (j == lane) mj = m[j];
        p.ws_m[ws_row(lane)] = mj;
        p.ws_l[ws_row(lane)] = Ls;
      }
    };

    int c = 0, qi = 0;
    for (; !stop; ++qi) {
      const int qs = qi & 1;
      warp_wait(&qfull[qs], (qi >> 1) & 1);
      stop = grp_sync_or(bad, grp);
      if (stop) break;
      const int32_t *us = unit_slots + qs * L::kUnitInts;
      const int nmem = us[3];
      // the previous unit first, while its statistics are still in m and l
      if (pend) {
        epilogue();
        pend = false;
        if (stop) break;
      }
      if (nmem == 0) break;  // the producer ran out of work
      const int ug = us[1], urow = us[2], nchunks = us[8];
      int ub[L::kSlots];
#pragma unroll
      for (int k = 0; k < L::kSlots; ++k) ub[k] = us[4 + k];
      const int32_t *ents = us + L::kUnitHead;  // -1 past the piece: those tokens are masked
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        m[j] = -INFINITY;
        l[j] = 0.f;
      }
      for (int ci = 0; ci < nchunks; ++ci, ++c) {
        float s[NC];
        warp_wait(&sfull[c & 1], (c >> 1) & 1);
        if (!bad) {
          tc::fence_after_sync();
          tc::tmem_ld16(trow + (c & 1) * N + c0, s);
        }
        const int32_t blk = ents[(ci * L::kChunk + r) >> log2_bs];
        const bool valid = blk >= 0 && blk < p.num_blocks;
        bool need = false;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          s[j] = (valid && !bad && col_valid(c0 + j, nmem)) ? s[j] * p.scale_log2 : -INFINITY;
          need |= s[j] > m[j] + kLazyRescale;
        }
        float mnew[NC];
        if (grp_sync_or(need || bad, grp)) {
          float *rm = red_at(red_max, c & 1);
          {  // this warp's max of every column; lane j (and j + 16) holds column j
            float v[NC];
#pragma unroll
            for (int j = 0; j < NC; ++j) v[j] = s[j];
            const float t = warp_reduce_columns<NC, true>(v, lane);
            if (lane < NC) rm[wq * NC + lane] = t;
          }
          stop = grp_sync_or(bad, grp);
          if (stop) break;
          const float4 *rm4 = reinterpret_cast<const float4 *>(rm);
#pragma unroll
          for (int j4 = 0; j4 < NC / 4; ++j4) {
            float4 cm = rm4[j4];
#pragma unroll
            for (int w = 1; w < 4; ++w) {
              const float4 x = rm4[w * (NC / 4) + j4];
              cm.x = fmaxf(cm.x, x.x);
              cm.y = fmaxf(cm.y, x.y);
              cm.z = fmaxf(cm.z, x.z);
              cm.w = fmaxf(cm.w, x.w);
            }
            mnew[4 * j4 + 0] = fmaxf(m[4 * j4 + 0], cm.x);
            mnew[4 * j4 + 1] = fmaxf(m[4 * j4 + 1], cm.y);
            mnew[4 * j4 + 2] = fmaxf(m[4 * j4 + 2], cm.z);
            mnew[4 * j4 + 3] = fmaxf(m[4 * j4 + 3], cm.w);
          }
        } else {
#pragma unroll
          for (int j = 0; j < NC; ++j) mnew[j] = m[j];
        }
        // weights of the old reference against the new one: 1 where it stays
        float alpha[NC];
        bool moved = false;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          moved |= mnew[j] != m[j];
          alpha[j] = (mnew[j] == m[j]) ? 1.f : ex2_approx(m[j] - mnew[j]);
        }
        if (moved && ci > 0) {
          // rescale the group's columns of the unit's O once PV(c-1) has
          // landed, before PV(c) adds
          warp_wait(&pvdone[(c - 1) & 1], ((c - 1) >> 1) & 1);
          if (!bad) {
            const uint32_t obuf = trow + 2 * N + (qi & 1) * N + c0;
            float o[NC];
            tc::fence_after_sync();
            tc::tmem_ld16(obuf, o);
#pragma unroll
            for (int k = 0; k < NC / 8; ++k) {
              float o8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) o8[e] = o[8 * k + e] * alpha[8 * k + e];
              tc::tmem_st8(obuf + 8 * k, o8);
            }
          }
        }
        // P(c) goes over P(c - 2), which PV(c - 2) must have read
        if (c >= 2) warp_wait(&pvdone[c & 1], ((c - 2) >> 1) & 1);
        __nv_bfloat16 *pb = reinterpret_cast<__nv_bfloat16 *>(smem + L::kOffP + (c & 1) * L::kP);
        const int kh = r >> 6, rr = r & 63;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int n = c0 + j;
          const float pv = s[j] == -INFINITY ? 0.f : ex2_approx(s[j] - mnew[j]);
          l[j] = fmaf(l[j], alpha[j], pv);
          m[j] = mnew[j];
          // P^T row n (K-major, 128-byte swizzle): token r in half kh
          const int off = kh * (N * 64) + (n >> 3) * 512 + (n & 7) * 64 + (((rr >> 3) ^ (n & 7)) << 3) + (rr & 7);
          pb[off] = __float2bfloat16_rn(pv);
        }
        fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(&pfull[c & 1]);
        if (ci == nchunks - 1 && r == 0) mbar_arrive(&qempty[qs]);  // one arrive per group
      }
      if (stop) break;
      pend = true;
      pun_g = ug;
      pun_row = urow;
      pun_nmem = nmem;
#pragma unroll
      for (int k = 0; k < L::kSlots; ++k) pun_b[k] = ub[k];
      p_clast = c - 1;
      p_u = qi;
    }
    if (stop) raise_error(PA_DEVERR_TIMEOUT);
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, L::kTmemCols);
}

}  // namespace pa

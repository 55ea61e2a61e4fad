// Paged chunked-prefill attention on the tensor cores (bf16, head_dim 128,
// group size 1..8).
//
// What it computes: for sequence b with len_b tokens in the cache, of which
// the last n_b are new (their queries are rows qstart[b] .. qstart[b+1]-1 of
// q), new token i at position p = len_b - n_b + i attends to the sequence's
// tokens 0..p through its block table ("PagedAttention Internals", "The Block
// Table Map"; "pagedattention" glossary entry, paragraph 3): the decode step
// of the same pages, for every new token, with a causal limit.  Written to
// out[qstart[b] + i][h][:], rounded once to bf16.
//
// How, on sm_100a (the flash-attention scheme with the pool behind a table):
//  * A work unit is (sequence, kv head, query tile): 128 query rows = Mq =
//    128 / G new tokens x the G query heads of the kv head, rows ordered
//    (token, head), loaded by one 3-D TMA box per column half.
//  * The unit walks 128-key chunks of its sequence up to its last token's
//    position.  Warp 0 (producer) loads each chunk's K and V tiles with one
//    4-D box per (block, kv head) as the decode kernel does; warp 1 issues
//        S[128 q x 128 keys] = Q . K^T              (M = N = 128, K = 128 d)
//        O[128 q x 128 d]   += P . V               (M = N = 128, K = 128 keys)
//    with S double-buffered and O double-buffered by unit in tensor memory;
//    the PV MMA takes P from tensor memory (A operand in TMEM).  Q tiles are
//    double-buffered in shared memory so the next unit's loads overlap.
//  * Warps 2..9, two halves of four warps: half h takes keys 64h .. 64h + 63
//    of every chunk and head-dim columns 64h .. 64h + 63 of O, and thread r
//    of a half owns query row r, so each row is shared by one warp of each
//    half (the pair of warps on the same tensor-memory lanes).  Per chunk a
//    thread reads its half of the row's S, masks keys past its position (per
//    32-key group), and weighs against a per-row reference max that moves
//    only when a score passes it by 2^8; the pair agrees on the reference
//    (and on any rescale of its O rows, each half rescaling its columns)
//    through one named barrier per chunk.  It writes its half of the row of
//    P in bf16 over the first half of its own S columns.  Each half keeps its
//    own sum of weights; at the end of a unit (overlapped with the next
//    unit) each half reads its columns of the row of O, divides by the sum
//    of both halves' sums and stores them.
//  * Every wait has a time limit (PA_DEVERR_TIMEOUT; the kernel drains and
//    frees tensor memory).  A table entry outside the pool is loaded as zeros
//    and sets PA_DEVERR_TABLE; that sequence's rows are then undefined.
#pragma once

#include "pa_decode_tc.cuh"

namespace pa {

struct PfLayout {
  static constexpr int kM = 128;           // query rows per tile
  static constexpr int kChunk = 128;       // keys per chunk
  static constexpr int kStages = 2;
  static constexpr int kTile = kChunk * 256;  // a K or V chunk: 128 keys x 256 B
  static constexpr int kGroup = 2048;         // 8 keys: two 1 KiB swizzle atoms (column halves)
  static constexpr int kHalf = kM * 128;      // a column (or key) half of a 128-row tile
  static constexpr int kMaxSeqs = 1024;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffQ = kOffV + kStages * kTile;  // two Q tiles of 2 column halves
  static constexpr int kQ = 2 * kHalf;
  static constexpr int kOffBar = kOffQ + 2 * kQ;
  static constexpr int kNumBars = 21;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  // unit slot: [b, g, first query row, tokens in the tile, first position, chunks, length]
  static constexpr int kUnitInts = 8;
  static constexpr int kOffUnit = kOffTmem + 16;
  static constexpr int kOffScan = kOffUnit + 2 * kUnitInts * 4;
  // row statistics the two softmax halves of a row exchange: [half][row]
  // maxima, and [unit parity][half][row] sums
  static constexpr int kOffXMax = kOffScan + 64;
  static constexpr int kOffXSum = kOffXMax + 2 * kM * 4;
  static constexpr int kOffPrefix = kOffXSum + 2 * 2 * kM * 4;  // tiles before each sequence
  static constexpr int kBytes = kOffPrefix + (kMaxSeqs + 1) * 4 + 1024;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;  // S0 S1 O0 O1, 128 columns each
};

struct PrefillParams {
  const int32_t *qstart;   // [B + 1]
  int32_t Mq;              // new tokens per query tile (128 / G)
};

template <int G>
__global__ void __launch_bounds__(PfLayout::kThreads, 1)
    prefill_tc(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
               const __grid_constant__ CUtensorMap tmap_q, DecodeParams p, PrefillParams pp) {
  using L = PfLayout;
  constexpr int Mq = L::kM / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *kfull = bars, *kempty = bars + 2, *vfull = bars + 4, *vempty = bars + 6;
  uint64_t *qfull = bars + 8, *qempty = bars + 10, *sfull = bars + 12, *pfull = bars + 14;
  uint64_t *pvdone = bars + 16, *ofree = bars + 18, *drain = bars + 20;
  int32_t *prefix = reinterpret_cast<int32_t *>(smem + L::kOffPrefix);
  int32_t *scan = reinterpret_cast<int32_t *>(smem + L::kOffScan);
  int32_t *unit_slots = reinterpret_cast<int32_t *>(smem + L::kOffUnit);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmem);
  __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(p.out);

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      // the MMA warp's commit after the unit's last QK + each of the four
      // softmax warps once it has read the unit (they run without a common
      // barrier, so every one must have passed its wait on qfull before the
      // slot and its barrier phase can be reused)
      mbar_init(&qempty[i], 1 + 8);
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 256);  // P of the chunk written over its S (both halves)
      mbar_init(&pvdone[i], 1);
      mbar_init(&ofree[i], 256);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }

  // query tiles of every sequence and their exclusive prefix sums (lengths
  // and query starts are caller data that no kernel of the library writes)
  const int B = p.B;
  constexpr int kMaxSeg = (L::kMaxSeqs + L::kThreads - 1) / L::kThreads;
  const int seg = (B + blockDim.x - 1) / blockDim.x;
  const int b_first = threadIdx.x * seg;
  int cnt[kMaxSeg];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < kMaxSeg; ++i) {
    cnt[i] = 0;
    const int b = b_first + i;
    if (i < seg && b < B) {
      const int n = pp.qstart[b + 1] - pp.qstart[b];
      const int ctx = p.lens[b];
      const bool ok = n >= 0 && n <= ctx && ctx <= p.max_ctx;
      if (!ok && blockIdx.x == 0) raise_error(PA_DEVERR_LEN);
      cnt[i] = ok ? (n + Mq - 1) / Mq : 0;
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
    const int b = b_first + i;
    if (i < seg && b < B) {
      prefix[b] = run;
      run += cnt[i];
      if (b == B - 1) prefix[B] = run;
    }
  }
  if (warp == 1) tc::tmem_relinquish();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int num_units = p.Hkv * prefix[B];
  uint32_t *sched = g_sched + 2 * p.sched_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tensormap(&tmap_k);
      tc::prefetch_tensormap(&tmap_v);
      tc::prefetch_tensormap(&tmap_q);
    }
    wait_prior_grid();  // the copies read the pool and q, which may be written just before
    allow_next_grid();
    const uint64_t pol_kv = tc::policy_evict_last();  // later tiles of the sequence read the same keys
    const uint64_t pol_q = policy_evict_first();
    const int bs = p.bs;
    const int bpc = L::kChunk / bs;  // blocks per chunk
    const int oob_group = p.num_blocks * p.Hkv * (bs / 8);
    int c = 0, qi = 0;
    bool ok = true;
    int u = blockIdx.x;
    while (ok && u < num_units) {
      // unit u: kv head u % Hkv of tile w = u / Hkv; tiles of a sequence in
      // descending order (the longest-reaching first)
      const int w = u / p.Hkv, g = u - (u / p.Hkv) * p.Hkv;
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= w) lo = mid; else hi = mid - 1;
      }
      const int b = lo;
      const int ntile = prefix[b + 1] - prefix[b];
      const int qt = ntile - 1 - (w - prefix[b]);
      const int q0 = pp.qstart[b];
      const int n = pp.qstart[b + 1] - q0;
      const int ctx = p.lens[b];
      const int tok0 = qt * Mq;
      const int ntok = min(Mq, n - tok0);
      const int pos0 = ctx - n + tok0;            // position of the tile's first token
      const int nchunks = (pos0 + ntok - 1) / L::kChunk + 1;
      const int32_t *tr = p.tables + (size_t)b * p.max_blocks;
      // this chunk's table entries: lane j < bpc holds block j of the chunk
      auto entry = [&](int ch) {
        const int j = ch * bpc + lane;
        return (lane < bpc && j * bs < ctx) ? tr[j] : -1;
      };
      int32_t e_next = entry(0);
      const int qs = qi & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&qempty[qs], ((qi >> 1) & 1) ^ 1))) { ok = false; break; }
      if (lane == 0) {
        int32_t *us = unit_slots + qs * L::kUnitInts;
        us[0] = b;
        us[1] = g;
        us[2] = q0 + tok0;
        us[3] = ntok;
        us[4] = pos0;
        us[5] = nchunks;
        us[6] = ctx;
        mbar_arrive_expect_tx(&qfull[qs], 2 * L::kHalf);
        uint8_t *qdst = smem + L::kOffQ + qs * L::kQ;
        tc::tma_load_3d(qdst, &tmap_q, 0, g * G, q0 + tok0, &qfull[qs], pol_q);
        tc::tma_load_3d(qdst + L::kHalf, &tmap_q, 64, g * G, q0 + tok0, &qfull[qs], pol_q);
      }
      ++qi;
      // chunk cc's K (which 0) or V (which 1) tiles, table entry e of this lane
      auto issue = [&](int cc, int ci_, int which, int32_t e) -> bool {
        const int slot = cc % L::kStages, use = cc / L::kStages;
        uint64_t *empty = which ? &vempty[slot] : &kempty[slot];
        uint64_t *full = which ? &vfull[slot] : &kfull[slot];
        const CUtensorMap *map = which ? &tmap_v : &tmap_k;
        if (!__all_sync(0xffffffffu, mbar_wait(empty, (use & 1) ^ 1))) return false;
        uint8_t *dst = smem + (which ? L::kOffV : L::kOffK) + slot * L::kTile;
        if (lane == 0) mbar_arrive_expect_tx(full, L::kTile);
        __syncwarp();
        if (lane < bpc) {
          int wq = oob_group;  // keys past the sequence: zeros (masked anyway)
          if (e >= 0 && e < p.num_blocks) wq = (e * p.Hkv + g) * (bs / 8);
          else if (which == 0 && (ci_ * bpc + lane) * bs < ctx) raise_error(PA_DEVERR_TABLE);
          tc::tma_load_4d(dst + lane * (bs / 8) * L::kGroup, map, 0, 0, 0, wq, full, pol_kv);
        }
        return true;
      };
      // K runs one chunk ahead of V: a K slot frees when its QK is done, a V
      // slot only when its PV is, after the chunk's softmax; so the next
      // chunk's K does not wait behind a V slot.
      int32_t e_prev = -1;
      for (int ci = 0; ci < nchunks; ++ci, ++c) {
        const int32_t e = e_next;
        if (!issue(c, ci, 0, e)) { ok = false; break; }
        if (ci > 0 && !issue(c - 1, ci - 1, 1, e_prev)) { ok = false; break; }
        e_prev = e;
        if (ci + 1 < nchunks) e_next = entry(ci + 1);
      }
      if (ok && !issue(c - 1, nchunks - 1, 1, e_prev)) ok = false;
      if (!ok) break;
      int raw = 0;
      if (lane == 0) raw = (int)gridDim.x + (int)atomicAdd(sched, 1u);
      u = __shfl_sync(0xffffffffu, raw, 0);
    }
    if (ok) {  // an empty unit stops the consumers
      const int qs = qi & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&qempty[qs], ((qi >> 1) & 1) ^ 1))) {
        ok = false;
      } else {
        if (lane == 0) unit_slots[qs * L::kUnitInts + 5] = 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfull[qs]);
      }
    }
    if (!ok && lane == 0) {
      raise_error(PA_DEVERR_TIMEOUT);
      for (int k = (c > L::kStages ? c - L::kStages : 0); k <= c; ++k) {
        mbar_wait(&kfull[k % L::kStages], (k / L::kStages) & 1, 100000000ull);
        mbar_wait(&vfull[k % L::kStages], (k / L::kStages) & 1, 100000000ull);
      }
      for (int k = (qi > 2 ? qi - 2 : 0); k < qi; ++k) mbar_wait(&qfull[k & 1], (k >> 1) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    wait_prior_grid();
    allow_next_grid();
    constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(128, 128, false, true);
    const uint32_t kbase0 = smem_u32(smem + L::kOffK), vbase0 = smem_u32(smem + L::kOffV);
    const uint32_t qbase0 = smem_u32(smem + L::kOffQ);
    bool ok = true;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    struct PvJob {
      int c, u;
      bool first;
    };
    auto issue_pv = [&](const PvJob &j) -> bool {
      const int c = j.c;
      if (!warp_wait(&pfull[c & 1], (c >> 1) & 1)) return false;
      if (!warp_wait(&vfull[c % L::kStages], (c / L::kStages) & 1)) return false;
      if (j.first && !warp_wait(&ofree[j.u & 1], ((j.u >> 1) & 1) ^ 1)) return false;
      if (lane == 0) {
        tc::fence_after_sync();
        const uint32_t vb = vbase0 + (c % L::kStages) * L::kTile;
        const uint32_t d = tmem + 256 + (j.u & 1) * 128;
        const uint32_t pa = tmem + (c & 1) * 128;  // P over the chunk's S columns, 2 keys per column
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // P: 16 keys = 8 columns of tensor memory; V: N = head dim
          // contiguous (MN-major), 16 keys = two 8-key groups
          const uint64_t bdesc = tc::smem_desc_sw128(vb + kk * 2 * L::kGroup, 1024, L::kGroup);
          // keys 0..63 in columns 0..31, keys 64..127 in columns 64..95 (each
          // softmax half writes its P over the first half of its own S columns)
          tc::mma_bf16_ts(d, pa + (kk >> 2) * 64 + (kk & 3) * 8, bdesc, idesc_pv, (kk > 0 || !j.first) ? 1u : 0u);
        }
        tc::mma_commit(&pvdone[c & 1]);
        tc::mma_commit(&vempty[c % L::kStages]);
      }
      __syncwarp();
      return true;
    };
    int c = 0, qi = 0;
    PvJob pending{-1, 0, false};
    while (ok) {
      const int qs = qi & 1;
      if (!warp_wait(&qfull[qs], (qi >> 1) & 1)) { ok = false; break; }
      const int nchunks = unit_slots[qs * L::kUnitInts + 5];
      if (nchunks == 0) break;
      const uint32_t qb = qbase0 + qs * L::kQ;
      for (int ci = 0; ci < nchunks; ++ci, ++c) {
        const int slot = c % L::kStages;
        if (!warp_wait(&kfull[slot], (c / L::kStages) & 1)) { ok = false; break; }
        if (lane == 0) {
          tc::fence_after_sync();
          const uint32_t kb = kbase0 + slot * L::kTile;
          const uint32_t d = tmem + (c & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // Q: K-major over the head dim (column half kk/4 at +kHalf);
            // K: K-major, 8-key groups kGroup apart, column half at +1 KiB
            const uint64_t a = tc::smem_desc_sw128(qb + (kk >> 2) * L::kHalf + (kk & 3) * 32, 16, 1024);
            const uint64_t bdesc = tc::smem_desc_sw128(kb + (kk >> 2) * 1024 + (kk & 3) * 32, 16, L::kGroup);
            tc::mma_bf16(d, a, bdesc, idesc_qk, kk > 0);
          }
          tc::mma_commit(&sfull[c & 1]);
          tc::mma_commit(&kempty[slot]);
          if (ci == nchunks - 1) tc::mma_commit(&qempty[qs]);
        }
        __syncwarp();
        if (pending.c >= 0 && !issue_pv(pending)) { ok = false; break; }
        pending = PvJob{c, qi, ci == 0};
      }
      ++qi;
    }
    if (ok && pending.c >= 0 && !issue_pv(pending)) ok = false;
    if (!ok && lane == 0) raise_error(PA_DEVERR_TIMEOUT);
    if (lane == 0) tc::mma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Two halves of four warps: half h (warps 2-5: h = 0; warps 6-9: h = 1)
    // takes keys 64h .. 64h + 63 of every chunk and head-dim columns
    // 64h .. 64h + 63 of O.  Thread r of a half owns query row r (its warp's
    // tensor-memory lane quadrant), so each row is held by one warp of each
    // half; the two warps of a quadrant form a pair that agrees, through
    // named barrier 1 + quadrant over their 64 threads, on the row's
    // reference and on stopping.  Each half keeps its own sum of weights over
    // its keys against the shared reference; the epilogue adds the two.
    wait_prior_grid();  // before the first write of out
    allow_next_grid();
    const int half = (warp - 2) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;            // query row: token r / G, head r % G
    const int pair_bar = 1 + wq;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    float *xmax = reinterpret_cast<float *>(smem + L::kOffXMax);  // [half][row]
    float *xsum = reinterpret_cast<float *>(smem + L::kOffXSum);  // [unit parity][half][row]
    bool bad = false;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      if (!bad && !__all_sync(0xffffffffu, mbar_wait(bar, parity))) bad = true;
    };
    // OR of pred over the pair's 64 threads; both warps of a pair take the
    // same sequence of these, so the pair never waits on a warp that left
    auto pair_or = [&](bool pred) {
      int res;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\t"
          "setp.ne.b32 p, %1, 0;\n\t"
          "bar.red.or.pred q, %2, 64, p;\n\t"
          "selp.s32 %0, 1, 0, q;\n\t}"
          : "=r"(res)
          : "r"((int)pred), "r"(pair_bar)
          : "memory");
      return res != 0;
    };
    float m = -INFINITY, l = 0.f;
    // the unit whose output is pending
    bool pend = false;
    int p_g = 0, p_row0 = 0, p_ntok = 0, p_clast = 0, p_u = 0;
    auto epilogue = [&]() {
      warp_wait(&pvdone[p_clast & 1], (p_clast >> 1) & 1);
      // the row's sum over both halves' keys (each half wrote its part at the
      // unit's end, before the pair's next barrier); the same order in both
      const float lrow = xsum[((p_u & 1) * 2 + 0) * L::kM + r] + xsum[((p_u & 1) * 2 + 1) * L::kM + r];
      const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
      const int tok = r / G, h = p_g * G + (r % G);
      const bool row_ok = tok < p_ntok && !bad;
      __nv_bfloat16 *dst = out + ((size_t)(p_row0 + tok) * p.Hq + h) * 128 + 64 * half;
      if (!bad) tc::fence_after_sync();
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float o[32];
        if (!bad) tc::tmem_ld32(trow + 256 + (p_u & 1) * 128 + 64 * half + 32 * k, o);
        if (row_ok) {
          uint4 v[4];
          uint32_t *w = reinterpret_cast<uint32_t *>(v);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 two = __floats2bfloat162_rn(o[2 * e] * inv, o[2 * e + 1] * inv);
            w[e] = *reinterpret_cast<const uint32_t *>(&two);
          }
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * k);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = v[e];
        }
      }
      tc::fence_before_sync();
      mbar_arrive(&ofree[p_u & 1]);
    };

    int c = 0, qi = 0;
    for (;; ++qi) {
      const int qs = qi & 1;
      warp_wait(&qfull[qs], (qi >> 1) & 1);
      if (pair_or(bad)) {
        bad = true;
        break;
      }
      const int32_t *us = unit_slots + qs * L::kUnitInts;
      const int nchunks = us[5];
      const int ug = us[1], urow0 = us[2], untok = us[3], upos0 = us[4], uctx = us[6];
      // keys of the sequence's last, partly filled block past its end
      const int tail_end = ((uctx + p.bs - 1) / p.bs) * p.bs;
      // the producer may reuse the Q tile once the QKs are done and every
      // softmax warp has read this unit's slot: it never runs two units
      // ahead of the slowest warp
      if (lane == 0 && nchunks > 0) mbar_arrive(&qempty[qs]);
      if (nchunks == 0) {
        if (pend) {
          asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");  // the partner's last sum is written
          epilogue();
        }
        break;
      }
      const int pos = upos0 + r / G;  // this row's position (rows past the tile's tokens: masked out)
      const bool row_live = r / G < untok;
      m = -INFINITY;
      l = 0.f;
      bool stop = false;
      for (int ci = 0; ci < nchunks; ++ci, ++c) {
        warp_wait(&sfull[c & 1], (c >> 1) & 1);
        if (!bad) tc::fence_after_sync();
        const uint32_t srow = trow + (c & 1) * 128 + 64 * half;  // this half's 64 columns of S
        const int key0 = ci * L::kChunk;
        // keys of this chunk the row sees (the first nrow), and of this half's
        const int nrow = row_live ? max(0, min(L::kChunk, pos - key0 + 1)) : 0;
        const int nvis = max(0, min(64, nrow - 64 * half));
        // One pass against the current reference: the weights stay in
        // registers until the pair knows that every row of its quadrant stays
        // within 2^8 of its reference; otherwise (a score past the bound in
        // either half) the chunk takes two passes:
        // the row max over both halves, a rescale of the rows' O, then the
        // weights.  Either way the weights are 2^(s - m) against the row's
        // reference m, the same in both halves.
        float s[32];
        uint32_t w[32];
        float lsum = 0.f;
        if (ci == 0 && !bad) {
          // A unit's first chunk: the row's reference starts at its score of
          // key 0 (visible to every row of the tile; both halves read the same
          // column, so they start from the same reference).  Scores within 2^8
          // of it keep the one pass; a larger one takes the two passes.  The
          // TMEM load is warp-wide (every lane takes part, live row or not).
          float s8[8];
          tc::tmem_ld8(trow + (c & 1) * 128, s8);
          if (row_live) m = s8[0] * p.scale_log2;
        }
        bool over = false;
        if (__all_sync(0xffffffffu, nvis == 64)) {
          // every row of the warp sees all of this half's keys (the chunks
          // before the diagonal): no masks, and one max instead of a test
          // per score
          float xmax = -INFINITY;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (!bad) tc::tmem_ld32(srow + 32 * k, s);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x0 = fmaf(s[2 * e], p.scale_log2, -m), x1 = fmaf(s[2 * e + 1], p.scale_log2, -m);
              xmax = fmaxf(xmax, fmaxf(x0, x1));
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              lsum += p0 + p1;
              const __nv_bfloat162 two = __floats2bfloat162_rn(p0, p1);
              w[16 * k + e] = *reinterpret_cast<const uint32_t *>(&two);
            }
          }
          over = xmax > kLazyRescale;
        } else {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (!bad) tc::tmem_ld32(srow + 32 * k, s);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x0 = fmaf(s[2 * e], p.scale_log2, -m), x1 = fmaf(s[2 * e + 1], p.scale_log2, -m);
              const bool v0 = 32 * k + 2 * e < nvis, v1 = 32 * k + 2 * e + 1 < nvis;
              over |= (v0 && x0 > kLazyRescale) || (v1 && x1 > kLazyRescale);
              const float p0 = v0 ? ex2_approx(x0) : 0.f, p1 = v1 ? ex2_approx(x1) : 0.f;
              lsum += p0 + p1;
              const __nv_bfloat162 two = __floats2bfloat162_rn(p0, p1);
              w[16 * k + e] = *reinterpret_cast<const uint32_t *>(&two);
            }
          }
        }
        if (!pair_or(over || bad)) {
          if (!bad) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              uint32_t w16[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) w16[e] = w[16 * k + e];
              tc::tmem_st16_nowait(srow + 16 * k, w16);
            }
            tc::tmem_wait_st();
          }
          l += lsum;
        } else {
          // pass 1: this half's max over its visible keys (base-2 units),
          // then the row's over both halves
          float cmax = -INFINITY;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (!bad) tc::tmem_ld32(srow + 32 * k, s);
            if (32 * k + 32 <= nvis) {
#pragma unroll
              for (int e = 0; e < 32; ++e) cmax = fmaxf(cmax, s[e] * p.scale_log2);
            } else if (32 * k < nvis) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (32 * k + e < nvis) cmax = fmaxf(cmax, s[e] * p.scale_log2);
            }
          }
          xmax[half * L::kM + r] = cmax;
          if (pair_or(bad)) {  // also makes both halves' maxima visible to the pair
            stop = true;
            break;
          }
          cmax = fmaxf(xmax[r], xmax[L::kM + r]);
          // the reference moves only when a score passes it by 2^8
          const bool need = cmax > m + kLazyRescale;
          const float mnew = need ? cmax : m;
          const float alpha = need ? exp2f(m - mnew) : 1.f;  // 0 when m was -inf
          if (__any_sync(0xffffffffu, need) && ci > 0) {
            // rescale this half's columns of the warp's O rows once PV(c-1)
            // has landed, before PV(c) adds
            warp_wait(&pvdone[(c - 1) & 1], ((c - 1) >> 1) & 1);
            if (!bad) {
              const uint32_t orow = trow + 256 + (qi & 1) * 128 + 64 * half;
              tc::fence_after_sync();
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                float o[32];
                tc::tmem_ld32(orow + 32 * k, o);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  float o8[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) o8[e] = o[8 * j + e] * alpha;
                  tc::tmem_st8(orow + 32 * k + 8 * j, o8);
                }
              }
            }
          }
          l *= alpha;
          m = mnew;
          // pass 2: P = 2^(s - m) in bf16, two keys per column, written over
          // columns 16k .. 16k + 15 of this half once group k of its S
          // (columns 32k ..) is read
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (!bad) tc::tmem_ld32(srow + 32 * k, s);
            float pv[32];
            if (32 * k + 32 <= nvis) {
#pragma unroll
              for (int e = 0; e < 32; ++e) pv[e] = ex2_approx(fmaf(s[e], p.scale_log2, -m));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                pv[e] = 32 * k + e < nvis ? ex2_approx(fmaf(s[e], p.scale_log2, -m)) : 0.f;
            }
            uint32_t w16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              l += pv[2 * e] + pv[2 * e + 1];
              const __nv_bfloat162 two = __floats2bfloat162_rn(pv[2 * e], pv[2 * e + 1]);
              w16[e] = *reinterpret_cast<const uint32_t *>(&two);
            }
            if (!bad) tc::tmem_st16_nowait(srow + 16 * k, w16);
          }
          if (!bad) tc::tmem_wait_st();
        }
        // V rows past the sequence's end in its last block hold whatever the
        // pool has there: zero them (thread r of the first half takes row r
        // of the chunk)
        const bool tail_row = half == 0 && key0 + r >= uctx && key0 + r < tail_end;
        if (half == 0 && __any_sync(0xffffffffu, tail_row)) {
          warp_wait(&vfull[c % L::kStages], (c / L::kStages) & 1);
          if (!bad && tail_row) {
            uint4 *vr = reinterpret_cast<uint4 *>(smem + L::kOffV + (c % L::kStages) * L::kTile +
                                                  (r >> 3) * L::kGroup + (r & 7) * 128);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              vr[e] = make_uint4(0, 0, 0, 0);
              vr[1024 / 16 + e] = make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
        }
        tc::fence_before_sync();
        mbar_arrive(&pfull[c & 1]);
        // the previous unit's rows, while this chunk's PV runs
        if (ci == 0 && pend) {
          epilogue();
          pend = false;
        }
      }
      if (stop) {
        bad = true;
        break;
      }
      // this half's sum of the unit's weights, for the epilogue
      xsum[((qi & 1) * 2 + half) * L::kM + r] = l;
      pend = true;
      p_g = ug;
      p_row0 = urow0;
      p_ntok = untok;
      p_clast = c - 1;
      p_u = qi;
    }
    if (bad) raise_error(PA_DEVERR_TIMEOUT);
  }

  if (p.late_wait) wait_prior_grid();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&sched[0], 0u);
      atomicExch(&sched[1], 0u);
    }
  }
  if (warp == 1) tc::tmem_dealloc(tmem, L::kTmemCols);
}

}  // namespace pa

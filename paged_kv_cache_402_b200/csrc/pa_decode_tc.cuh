// Paged decode attention on the 5th-generation tensor cores (bf16, head_dim
// 128, group size 1..8): the split-context partition kernel.
//
// What it computes is what decode_partition_simt computes (see there for the
// pages it follows): for every (sequence b, kv head g, 512-token partition p)
// it reads keys and values through the block table, scores all G query heads
// of the group at once, runs an online softmax in base-2 units and writes
// either the final output (single-partition sequences) or the partition's
// (max, sum, unnormalised accumulator) for the log-sum-exp reduce.
//
// How, on sm_100a:
//  * Persistent grid, one CTA per SM.  Work units are in largest-first order
//    (every full 512-token partition, then the partial last partition of each
//    sequence); CTA i starts with unit i and then draws the next free unit
//    from a counter once the copies of its current unit are issued, so CTAs
//    that drew short units take more of them and all finish together.  The counter lives in one of kSchedSlots library-owned
//    slots, chosen per call, and the last CTA out resets it.
//  * Warp 6, on batches of mostly whole partitions, is the scheduler: it
//    draws the CTA's next unit, looks it up and loads its table entries
//    while the producer issues the current unit's copies, and hands the
//    description over through a one-slot queue in shared memory.  On
//    batches of mostly short tails the producer does that itself (the
//    scheduler's lookups would take issue slots from the softmax warp that
//    shares its sub-partition, once per short unit).
//  * Warp 0 is the TMA producer.  A unit is cut into chunks of 128 tokens;
//    each lane loads one block of a chunk: the whole (block, kv head) K tile,
//    and then the V tile, with ONE 4-D box each (a TMA issue costs about
//    90 ns per instruction per thread whatever its size, so the box is as big
//    as a tile and the lanes issue in parallel).  The 4-D view (64 columns,
//    8 rows, 2 column halves, 8-row groups) lands every tile in shared memory
//    as [8-row group][column half][8 rows x 128 B] with 128-byte swizzle:
//    each (group, half) is one swizzle atom, so the MMA sees uniform strides.
//    K and V go to 3-slot rings of 32 KiB slots.  Missing blocks (past the
//    partition, or a table entry outside the pool) are loaded from groups
//    past the end of the tensor, which the TMA fills with zeros.
//  * Warp 1 (one lane) issues tcgen05 MMAs: per chunk c,
//        S^T[128 tok x 16] = K_c[128 tok x 128 d] . Q^T[128 d x 16]   (K-major A and B)
//        O^T[128 d x 16]   = V_c^T[128 d x 128 tok] . P^T[128 tok x 16] (MN-major A)
//    with accumulators in tensor memory; the Q tile is the 16 query rows
//    from the group's first, one 3-D box (N = 16 is the smallest N an
//    M = 128 MMA takes; columns past G are not read).  S is double-buffered
//    by chunk; O is one accumulator per unit that every PV of the unit adds
//    to, double-buffered by unit so a unit's output is read while the next
//    one runs.  QK of chunk c is issued before PV of chunk c-1.
//  * Warps 2..5 (128 threads) run the softmax on S (thread = token row) and
//    write P^T in bf16 to shared memory.  The weights are taken against a
//    reference max that moves only when a score passes it by 2^8; when it
//    moves, the same threads (now thread = head-dim row) rescale the unit's O
//    in tensor memory before the next PV adds to it.  At the end of a unit
//    (overlapped with the first chunk of the next one) they read O and write
//    the output or the partition's statistics.
//  * Fused step (k_new set): the unit that holds a sequence's newest token
//    (its last partition, once per kv head) loads the sequence's last block
//    from the copy-on-write source when there is one (the rows before the
//    new one are the same); the MMA warp writes the new key/value row into
//    the landed K and V tiles before the MMAs read them, and stores it to
//    the pool; the softmax threads copy the source tile over the
//    destination (loads at the unit's start, stores once its first chunk's
//    weights are out).  No copy of this call reads what those stores write,
//    so nothing waits for them.
//  * Every mbarrier wait has an iteration limit; a thread that gives up sets
//    PA_DEVERR_TIMEOUT and its role stops, the softmax warps leave together
//    through a reducing barrier, the MMA lane drains its MMAs, and the CTA
//    frees its tensor memory before returning.
#pragma once

#include "pa_decode_simt.cuh"
#include "pa_tc.cuh"

namespace pa {

struct TcLayout {
  static constexpr int kN = 16;             // MMA N: the group's query heads, then the next rows
                                            // (M = 128 takes N in multiples of 16)
  static constexpr int kChunk = 128;        // tokens per MMA chunk (= M)
  static constexpr int kStages = 3;
  static constexpr int kTile = kChunk * 256;  // 128 tokens x 256 B = 32 KiB
  static constexpr int kGroup = 2048;         // one 8-row group: two 1 KiB swizzle atoms (column halves)
  static constexpr int kQ = 2 * kN * 128;     // two halves of kN rows x 128 B
  static constexpr int kP = 2 * kN * 128;     // two 64-token halves of kN rows x 128 B
  static constexpr int kMaxSeqs = 1024;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffQ = kOffV + kStages * kTile;
  static constexpr int kOffP = kOffQ + 2 * kQ;
  static constexpr int kOffBar = kOffP + 2 * kP;
  static constexpr int kNumBars = 27;
  static constexpr int kOffRed = kOffBar + (kNumBars * 8 + 15) / 16 * 16;  // 16-byte aligned
  static constexpr int kRedFloats = 2 * 4 * kN;  // [parity][warp][head]
  static constexpr int kOffRedSum = kOffRed + kRedFloats * 4;
  static constexpr int kOffTmem = kOffRedSum + kRedFloats * 4;
  // per-unit description written by the producer next to the unit's Q slot:
  // [b, g, part, t0, t1, nchunks, single, newest-token block or -1,
  //  copy-on-write source of that block or -1, packed] + the unit's table
  // entries (as the copies read them)
  static constexpr int kUnitHead = 10;
  static constexpr int kMaxPart = 1024;  // the largest partition built (256, 512 or 1024 tokens)
  static constexpr int kUnitInts = kUnitHead + kMaxPart / 8;
  static constexpr int kOffUnit = kOffTmem + 16;
  static constexpr int kOffScan = kOffUnit + 2 * kUnitInts * 4;  // 4 x 8 ints
  // head-packed passes: each warp's column maxima (by chunk parity) and
  // weights of the old reference, and the pending unit's maxima (by unit
  // parity), 16 columns each
  static constexpr int kOffPack = kOffScan + 128;
  static constexpr int kOffPrefix = kOffPack + 3 * 2 * kN * 4;
  static constexpr int kOffCtx = kOffPrefix + (kMaxSeqs + 1) * 4;
  static constexpr int kOffFirst = kOffCtx + kMaxSeqs * 4;  // first partition of each sequence
  // the next unit's description, from the scheduler warp to the producer:
  // [valid, b, g, part, t0, t1, nchunks, hg, single, pack, nd, ns, -, -, -, -]
  // + the unit's table entries
  static constexpr int kDescHead = 16;
  static constexpr int kOffDesc = kOffFirst + kMaxSeqs * 4;
  static constexpr int kBytes = kOffDesc + (kDescHead + kMaxPart / 8) * 4 + 1024;  // + alignment slack
  static constexpr int kThreads = 224;
  static constexpr uint32_t kTmemCols = 64;  // S0 S1 O0 O1, kN columns each
};
static_assert(TcLayout::kBytes <= 227 * 1024, "shared memory of the partition kernel");

// Head packing of short partial partitions (group size <= 4, a multiple of 4
// kv heads): one pass covers 4 kv heads of a sequence, with 32 rows of the
// 128-row K and V tiles per head, so that a head's rows are one softmax
// warp's.  Its query tile holds the 4 G query rows of the 4 heads (adjacent
// in q), S and O are block diagonal: a score counts only where the row's
// head is the column's.
constexpr int kPackHeads = 4;
constexpr int kPackRows = TcLayout::kChunk / kPackHeads;

// 2^x by the MUFU approximation (flushes denormal results to zero): the
// weights only feed a bf16 operand and fp32 sums.  Every tensor-core kernel
// takes its softmax weights with it, so that the cascade and the partition
// kernel give the same statistics for the same tiles.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Reduces NC columns held by every lane of a warp (v[n]: this lane's value
// of column n) and returns column (lane % NC)'s result.  Lanes differing in
// bit 4, then 3, ... down to bit log2(NC) are combined over all columns; then
// each further step hands half of the remaining columns to the partner lane
// (lane ^ NC/2, ..., lane ^ 1) and combines the other half with the
// partner's.  NC log2(32 / NC) + NC - 1 shuffles instead of 5 NC.  A sum is
// taken over the same pairs in the same order as a butterfly per column
// (bit 4 first, ..., bit 0), so it has the same bits.  v is consumed.
template <int NC, bool kMax>
__device__ __forceinline__ float warp_reduce_columns(float (&v)[NC], int lane) {
  static_assert(NC >= 1 && NC <= 32 && (NC & (NC - 1)) == 0, "columns");
#pragma unroll
  for (int off = 16; off >= NC; off >>= 1) {
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const float recv = __shfl_xor_sync(0xffffffffu, v[i], off);
      v[i] = kMax ? fmaxf(v[i], recv) : v[i] + recv;
    }
  }
#pragma unroll
  for (int off = NC / 2; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

// Combines the four warps' partial results of columns 0..NC-1 (red[w * ld + n],
// 16-byte aligned rows) in warp order: out[n] = op(...op(op(init, red[n]),
// red[ld + n])..., red[3 ld + n]).
template <int NC, bool kMax>
__device__ __forceinline__ void combine_warps(const float *red, int ld, float init, float (&out)[NC]) {
#pragma unroll
  for (int n = 0; n < NC; ++n) out[n] = init;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    if constexpr (NC % 4 == 0) {
#pragma unroll
      for (int n4 = 0; n4 < NC / 4; ++n4) {
        const float4 x = reinterpret_cast<const float4 *>(red + w * ld)[n4];
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) out[4 * n4 + k] = kMax ? fmaxf(out[4 * n4 + k], xs[k]) : out[4 * n4 + k] + xs[k];
      }
    } else {
#pragma unroll
      for (int n = 0; n < NC; ++n) out[n] = kMax ? fmaxf(out[n], red[w * ld + n]) : out[n] + red[w * ld + n];
    }
  }
}

// Largest excess (base-2 units) of a score over the running reference before
// the reference is moved: weights then stay below 2^8, far inside the range
// of the bf16 P operand and the fp32 sums.
constexpr float kLazyRescale = 8.0f;

struct TcUnit {
  int b, g, part, t0, t1, nchunks;
  int ctx;  // the sequence's length
  int hg;  // kv heads of the unit: g .. g + hg - 1 (1 for a full partition)
  bool single;
  bool pack;  // passes of kPackHeads heads, kPackRows tokens per head per chunk
};

// Run-time work counters: [next unit, CTAs finished] per slot.  A call takes
// slot (ticket % kSchedSlots); the last CTA of the call puts both back to 0,
// so the slot is ready for the call that takes it next.
constexpr int kSchedSlots = 64;
__device__ uint32_t g_sched[2 * kSchedSlots];

// prefix[b] packs, for sequences before b, the number of full 512-token
// partitions (bits 0..19) and of partial last partitions (bits 20..31).
constexpr int kFullBits = 20;
__device__ __forceinline__ int pf_of(int32_t v) { return v & ((1 << kFullBits) - 1); }
__device__ __forceinline__ int pp_of(int32_t v) { return (int)((uint32_t)v >> kFullBits); }

// Launches of more than TcLayout::kMaxSeqs sequences (up to kCoarse times
// that) take the kernel's COARSE form: for entries of kCoarse consecutive
// sequences, the prefix sums of their full partitions (prefix) and of their
// partial last ones (pprefix, where ctx_s is in the other form), unpacked;
// a lookup finds the entry, then the sequence from its members' lengths,
// one lane each.  One launch then covers a whole batch of a few thousand
// sequences.
constexpr int kCoarse = 8;

// Sequence b's length, first token (as validated: 0 unless a whole number
// of blocks inside the sequence), and its full partitions (from the one its
// first token falls in) and partial last one.
template <int PART>
__device__ __forceinline__ void seq_counts(const DecodeParams &p, int b, int &ctx, int &ft, int &nfull,
                                           int &npart) {
  ctx = p.lens[b];
  ft = p.first_tok ? p.first_tok[b] : 0;
  const bool ok = ctx >= 0 && ctx <= p.max_ctx;
  if (ft != 0 && (!ok || ft < 0 || ft >= ctx || ft % p.bs != 0)) ft = 0;
  const bool own = ok && ctx > 0;
  nfull = own ? ctx / PART - ft / PART : 0;
  npart = own && ctx % PART != 0 ? 1 : 0;
}

// Unit u of the largest-first order.  The full partitions (sequence-major,
// kv head fastest; a sequence's first one is the partition its first token
// first_s[b] falls in, which then starts at that token) are one kv head each; the partial last partitions are tail_hg consecutive kv heads of
// one sequence each (Hkv / tail_hg units per sequence).  With one head per
// tail unit the full partitions come first (units [0, F)), the partial ones
// after; with several heads a tail unit is about as large as a full one or
// larger, so the tail units come first (units [0, T)) and the full ones
// after, and a launch ends on units of one full partition either way.  With
// pack_ok (tail_hg then a multiple of kPackHeads), a tail unit goes in
// head-packed passes when they take fewer chunks in all.
// Called by a whole warp with the same u (a coarse lookup shares the work).
template <int PART, bool COARSE>
__device__ __forceinline__ TcUnit tc_unit_at(const DecodeParams &p, const int32_t *prefix,
                                             const int32_t *ctx_s, const int32_t *first_s, int u,
                                             int num_full, int num_tail, int tail_hg, bool pack_ok,
                                             int n_ent) {
  TcUnit un;
  const bool tails_first = tail_hg > 1;
  const bool full = tails_first ? u >= num_tail : u < num_full;
  const int v = full ? (tails_first ? u - num_tail : u) : (tails_first ? u : u - num_full);
  const int per_seq = full ? p.Hkv : p.Hkv / tail_hg;
  const int w = v / per_seq;
  un.hg = full ? 1 : tail_hg;
  un.g = (v - w * per_seq) * un.hg;
  int ctx, first, before;  // before: the unit's kind of partitions ahead of its sequence's
  if constexpr (!COARSE) {
    int lo = 0, hi = p.B - 1;  // largest b whose count before it is <= w
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      const int cnt = full ? pf_of(prefix[mid]) : pp_of(prefix[mid]);
      if (cnt <= w) lo = mid; else hi = mid - 1;
    }
    un.b = lo;
    ctx = ctx_s[lo];
    first = first_s[lo];
    before = pf_of(prefix[lo]);
  } else {
    const int32_t *pre = full ? prefix : ctx_s;  // the full / partial prefix sums
    int lo = 0, hi = n_ent - 1;  // largest entry whose count before it is <= w
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= w) lo = mid; else hi = mid - 1;
    }
    // lane i < kCoarse: the entry's i-th sequence, its count of the unit's kind
    const int lane = threadIdx.x & 31, i = lane & (kCoarse - 1);
    const int b = lo * kCoarse + i;
    int c = 0, sctx = 0, sft = 0, nf = 0, np = 0;
    if (lane < kCoarse && b < p.B) {
      seq_counts<PART>(p, b, sctx, sft, nf, np);
      c = full ? nf : np;
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < kCoarse; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o, kCoarse);
      if (i >= o) incl += t;
    }
    const int rel = w - pre[lo];
    const unsigned hit = __ballot_sync(0xffffffffu, lane < kCoarse && incl - c <= rel && rel < incl);
    const int src = hit ? __ffs(hit) - 1 : 0;
    un.b = lo * kCoarse + src;
    ctx = __shfl_sync(0xffffffffu, sctx, src);
    first = __shfl_sync(0xffffffffu, sft, src);
    before = pre[lo] + __shfl_sync(0xffffffffu, incl - c, src);
  }
  un.ctx = ctx;
  un.part = full ? first / PART + w - before : ctx / PART;
  un.t0 = max(un.part * PART, first);
  un.t1 = min((un.part + 1) * PART, ctx);
  const int len = un.t1 - un.t0;
  const int nc_plain = (len + TcLayout::kChunk - 1) / TcLayout::kChunk;
  const int nc_pack = (len + kPackRows - 1) / kPackRows;
  un.pack = pack_ok && !full && nc_pack < kPackHeads * nc_plain;
  un.nchunks = un.pack ? nc_pack : nc_plain;
  un.single = ctx <= PART && first == 0;
  return un;
}

// c ? a : b as one selp the compiler keeps: a chain of these over a small
// register array stays in registers (a plain ?: chain may be turned back
// into an indexed load from local memory).
__device__ __forceinline__ int32_t select_i32(bool c, int32_t a, int32_t b) {
  int32_t r;
  asm("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\tselp.b32 %0, %1, %2, q;\n\t}"
      : "=r"(r)
      : "r"(a), "r"(b), "r"((int)c));
  return r;
}

// OR of `pred` over the 128 softmax threads (named barrier 1).
__device__ __forceinline__ bool wg_sync_or(int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred)
      : "memory");
  return r != 0;
}

// PART: tokens per partition (256, 512 or 1024); the caller's p.part.
template <int G, int PART, bool COARSE>
__global__ void __launch_bounds__(TcLayout::kThreads, 1)
    decode_partition_tc(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v,
                        const __grid_constant__ CUtensorMap tmap_q, DecodeParams p) {
  using L = TcLayout;
  constexpr int N = L::kN;
  static_assert(G >= 1 && G <= N, "group size");
  static_assert(PART == 256 || PART == 512 || PART == 1024, "partition size");
  constexpr int NE = PART / 8 / 32;  // table entries per lane of a unit (bs >= 8)
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  // tmap_q: q in boxes of kN rows and both column halves.  A unit's tile
  // takes the kN query rows from its group's first one: the group's G (or a
  // head-packed pass's kPackHeads * G), then the next heads' (or the zero
  // fill past the end), whose S and O columns nothing reads.
  constexpr bool kCanPack = G <= 4;
  const bool pack_ok = kCanPack && p.Hkv % kPackHeads == 0;
  // Up to the first unit's table entries, the kernel reads only the lengths
  // and the block tables, which no kernel of this library writes; it waits
  // for the kernel ahead of it in the stream (and lets the next one be
  // scheduled) only after that, so this start-up overlaps the previous
  // kernel.  Each thread waits before it triggers.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *kfull = bars, *kempty = bars + 3, *vfull = bars + 6, *vempty = bars + 9;
  uint64_t *qfull = bars + 12, *qempty = bars + 14, *sfull = bars + 16, *pfull = bars + 18;
  uint64_t *pvdone = bars + 20, *ofree = bars + 22, *drain = bars + 24;
  uint64_t *dfull = bars + 25, *dempty = bars + 26;  // the description slot
  int32_t *desc = reinterpret_cast<int32_t *>(smem + L::kOffDesc);
  int32_t *prefix = reinterpret_cast<int32_t *>(smem + L::kOffPrefix);
  int32_t *ctx_s = reinterpret_cast<int32_t *>(smem + L::kOffCtx);
  int32_t *first_s = reinterpret_cast<int32_t *>(smem + L::kOffFirst);
  int32_t *scan = reinterpret_cast<int32_t *>(smem + L::kOffScan);
  int32_t *unit_slots = reinterpret_cast<int32_t *>(smem + L::kOffUnit);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmem);
  float *red_max = reinterpret_cast<float *>(smem + L::kOffRed);
  float *red_sum = reinterpret_cast<float *>(smem + L::kOffRedSum);
  float *pk_alpha = reinterpret_cast<float *>(smem + L::kOffPack);         // [parity][16]
  float *pk_mdone = pk_alpha + 2 * N;                                       // [parity][16]
  __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(p.out);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 2);  // the MMA lane's commit + the softmax warpgroup
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 128);
      mbar_init(&pvdone[i], 1);  // per chunk parity: the PV MMA of the chunk completed
      mbar_init(&ofree[i], 128);  // per unit parity: the epilogue read the unit's O
    }
    mbar_init(drain, 1);
    mbar_init(dfull, 1);
    mbar_init(dempty, 1);
    fence_barrier_init();
  }
  // The P tiles start zero (a plain unit only reads columns 0 .. G - 1 of S
  // and O, so what its Q tile holds past row G, and what a head-packed pass
  // leaves in the other rows of P, does not reach its output)
  for (int i = threadIdx.x; i < (2 * L::kQ + 2 * L::kP) / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(smem + L::kOffQ)[i] = make_uint4(0, 0, 0, 0);

  // partition counts of every sequence (COARSE: of every entry of kCoarse
  // sequences) and their exclusive prefix sums
  const int B = p.B;
  const int n_ent = COARSE ? (B + kCoarse - 1) / kCoarse : B;
  if constexpr (!COARSE) {
    constexpr int kMaxSeg = (L::kMaxSeqs + L::kThreads - 1) / L::kThreads;
    const int seg = (B + blockDim.x - 1) / blockDim.x;
    const int b_first = threadIdx.x * seg;
    int cnt[kMaxSeg];
    int mine = 0;
    // chunks of this thread's partial last partitions (128-token chunks, and
    // kPackRows-token ones of a packed pass), and their count
    int tail_chunks = 0, tail_pchunks = 0, tails = 0;
#pragma unroll
    for (int i = 0; i < kMaxSeg; ++i) {
      cnt[i] = 0;
      const int b = b_first + i;
      if (i < seg && b < B) {
        const int ctx = p.lens[b];
        const bool ok = ctx >= 0 && ctx <= p.max_ctx;
        // tokens the cascade kernel did: a whole number of blocks before the last
        int ft = p.first_tok ? p.first_tok[b] : 0;
        if (ft != 0 && (!ok || ft < 0 || ft >= ctx || ft % p.bs != 0)) {
          if (blockIdx.x == 0) raise_error(PA_DEVERR_PLAN);
          ft = 0;  // this kernel then does the whole sequence
        }
        if (ok && ctx % PART != 0) {
          const int tl = ctx - max(ctx / PART * PART, ft);
          tail_chunks += (tl + TcLayout::kChunk - 1) / TcLayout::kChunk;
          tail_pchunks += (tl + kPackRows - 1) / kPackRows;
          ++tails;
        }
        ctx_s[b] = ctx;
        first_s[b] = ft;
        // partitions from the one token ft falls in: the ones that end on a
        // partition boundary in the low bits, a partial last one in the high ones
        cnt[i] = (ok && ctx > 0) ? (ctx / PART - ft / PART) | ((ctx % PART != 0 ? 1 : 0) << kFullBits) : 0;
        mine += cnt[i];
        if (blockIdx.x == 0 && !ok) raise_error(PA_DEVERR_LEN);
      }
    }
    int incl = mine;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) scan[warp] = incl;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      tail_chunks += __shfl_xor_sync(0xffffffffu, tail_chunks, o);
      tail_pchunks += __shfl_xor_sync(0xffffffffu, tail_pchunks, o);
      tails += __shfl_xor_sync(0xffffffffu, tails, o);
    }
    if (lane == 0) {
      scan[8 + warp] = tail_chunks;
      scan[16 + warp] = tails;
      scan[24 + warp] = tail_pchunks;
    }
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
  } else {
    constexpr int kMaxSeg = (L::kMaxSeqs + L::kThreads - 1) / L::kThreads;
    const int seg = (n_ent + blockDim.x - 1) / blockDim.x;
    const int e_first = threadIdx.x * seg;
    int cnt[kMaxSeg], cntp[kMaxSeg];
    int mine = 0, minep = 0;
    int tail_chunks = 0, tail_pchunks = 0, tails = 0;
#pragma unroll
    for (int i = 0; i < kMaxSeg; ++i) {
      cnt[i] = cntp[i] = 0;
      const int e = e_first + i;
      if (i < seg && e < n_ent) {
#pragma unroll
        for (int k = 0; k < kCoarse; ++k) {
          const int b = e * kCoarse + k;
          if (b < B) {
            int ctx, ft, nf, np;
            seq_counts<PART>(p, b, ctx, ft, nf, np);
            if (blockIdx.x == 0 && p.first_tok && p.first_tok[b] != ft) raise_error(PA_DEVERR_PLAN);
            if (blockIdx.x == 0 && !(ctx >= 0 && ctx <= p.max_ctx)) raise_error(PA_DEVERR_LEN);
            if (np) {
              const int tl = ctx - max(ctx / PART * PART, ft);
              tail_chunks += (tl + TcLayout::kChunk - 1) / TcLayout::kChunk;
              tail_pchunks += (tl + kPackRows - 1) / kPackRows;
              ++tails;
            }
            cnt[i] += nf;
            cntp[i] += np;
          }
        }
        mine += cnt[i];
        minep += cntp[i];
      }
    }
    int incl = mine, inclp = minep;  // inclusive scans within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      const int vp = __shfl_up_sync(0xffffffffu, inclp, o);
      if (lane >= o) {
        incl += v;
        inclp += vp;
      }
    }
    // the warps' partial-count totals go to first_s[8 ..] (first_s is not
    // used in this form; the partial prefix sums reach first_s[0] at most)
    if (lane == 31) {
      scan[warp] = incl;
      first_s[8 + warp] = inclp;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      tail_chunks += __shfl_xor_sync(0xffffffffu, tail_chunks, o);
      tail_pchunks += __shfl_xor_sync(0xffffffffu, tail_pchunks, o);
      tails += __shfl_xor_sync(0xffffffffu, tails, o);
    }
    if (lane == 0) {
      scan[8 + warp] = tail_chunks;
      scan[16 + warp] = tails;
      scan[24 + warp] = tail_pchunks;
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, L::kTmemCols);
    __syncthreads();
    int run = incl - mine, runp = inclp - minep;
    for (int w = 0; w < warp; ++w) {
      run += scan[w];
      runp += first_s[8 + w];
    }
    int32_t *pprefix = ctx_s;
#pragma unroll
    for (int i = 0; i < kMaxSeg; ++i) {
      const int e = e_first + i;
      if (i < seg && e < n_ent) {
        prefix[e] = run;
        pprefix[e] = runp;
        run += cnt[i];
        runp += cntp[i];
        if (e == n_ent - 1) {
          prefix[n_ent] = run;
          pprefix[n_ent] = runp;
        }
      }
    }
  }
  if (warp == 1) tc::tmem_relinquish();
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int full_total = COARSE ? prefix[n_ent] : pf_of(prefix[B]);
  const int part_total = COARSE ? ctx_s[n_ent] : pp_of(prefix[B]);
  const int num_full = p.Hkv * full_total;
  // A partial last partition of a few chunks is a short unit, and a unit's
  // scheduling (the draw, the unit's lookup, its table entries) is a serial
  // chain of the producer; so the partial partitions of one sequence go out
  // tail_hg kv heads per unit, about a full partition's worth of chunks (the
  // same table entries serve every head).  Every CTA takes the same
  // decision from the same lengths; a launch keeps at least 4 units per CTA.
  int tail_hg = 1;
  {
    int tc_sum = 0, tp_sum = 0, tn = 0;
    for (int w = 0; w < L::kThreads / 32; ++w) {
      tc_sum += scan[8 + w];
      tn += scan[16 + w];
      tp_sum += scan[24 + w];
    }
    if (tn > 0 && tc_sum > 0) {
      // kv heads per unit: a full partition's chunks over the mean tail's,
      // rounded; with packing, packed passes of kPackHeads heads over the
      // mean packed pass's chunks
      const int step = pack_ok ? kPackHeads : 1;
      const int per = pack_ok ? tp_sum : tc_sum;
      int h = step * max((2 * (PART / L::kChunk) * tn + per) / (2 * per), 1);
      h = min(h, p.Hkv);
      while (h > step && (p.Hkv % h != 0 || num_full + (p.Hkv / h) * tn < 4 * (int)gridDim.x)) h -= step;
      tail_hg = h;
    } else if (pack_ok) {
      tail_hg = kPackHeads;
    }
  }
  const int num_tail = (p.Hkv / tail_hg) * part_total;
  const int num_units = num_full + num_tail;
  // Batches of mostly whole partitions: a scheduler warp draws and looks up
  // the units, so the producer's chain per unit holds only its copies.  On
  // batches of mostly short tails its lookups would take issue slots from
  // the softmax warp beside it on every unit; there the producer does them
  // itself.  Every CTA takes the same decision from the same counts.
  const bool use_sched = (int64_t)num_full * (PART / L::kChunk) >= 4 * (int64_t)num_tail;
  uint32_t *sched = g_sched + 2 * p.sched_slot;
  const int bs = p.bs;
  const int lg_bs = bs == 8 ? 3 : (bs == 16 ? 4 : 5);
  // A unit's table entries (at most PART / 8), entry 32 k + lane in
  // x[k] of the lane, loaded right after the previous unit's copies are
  // issued.  In a fused step a unit that holds its sequence's newest token
  // (position t1 - 1) also gets that token's block nd and the block ns to
  // copy over it (-1: none); its loads then read the last block from ns.
  auto pick = [](const int32_t (&x)[NE], int k) {  // x[k] by selects, never a local-memory index
    int32_t v = x[0];
#pragma unroll
    for (int i = 1; i < NE; ++i) v = select_i32(k == i, x[i], v);
    return v;
  };
  auto load_entries = [&](int u, TcUnit &nu, int32_t (&x)[NE], int32_t &nd, int32_t &ns) {
#pragma unroll
    for (int k = 0; k < NE; ++k) x[k] = -1;
    nd = ns = -1;
    if (u < num_units) {
      nu = tc_unit_at<PART, COARSE>(p, prefix, ctx_s, first_s, u, num_full, num_tail, tail_hg, pack_ok, n_ent);
      const int32_t *tr = p.tables + (size_t)nu.b * p.max_blocks + (nu.t0 >> lg_bs);
      const int nb = (nu.t1 - nu.t0 + bs - 1) >> lg_bs;
      const bool newest = p.k_new != nullptr && nu.t1 == nu.ctx;
      const int32_t src = (newest && p.cow_src != nullptr) ? p.cow_src[nu.b] : -1;
#pragma unroll
      for (int k = 0; k < NE; ++k)
        if (lane + 32 * k < nb) x[k] = tr[lane + 32 * k];
      if (newest) {
        const int jl = (nu.t1 - 1 - nu.t0) >> lg_bs;
        const int32_t blk = __shfl_sync(0xffffffffu, pick(x, jl >> 5), jl & 31);
        if (blk >= 0 && blk < p.num_blocks) {  // else its copy flags PA_DEVERR_TABLE
          nd = blk;
          if (src >= p.num_blocks) {
            if (lane == 0) raise_error(PA_DEVERR_PAIR);
          } else if (src >= 0) {
            ns = src;
#pragma unroll
            for (int k = 0; k < NE; ++k) x[k] = select_i32(lane == (jl & 31) && k == (jl >> 5), src, x[k]);
          }
        }
      }
    }
  };

  if (warp == 6) {
    // ------------------------------------------------------------ scheduler
    // Draws the CTA's units (the first is fixed, later ones come from the
    // call's work counter), looks each up and loads its table entries, and
    // hands the description to the producer through the one-slot queue, so
    // the producer's chain per unit holds only its copies.  The lookups read
    // the lengths, tables and copy sources, which no kernel of the library
    // writes.
    int u = blockIdx.x, di = 0;
    bool okq = true, first = true;
    for (; use_sched;) {
      TcUnit nu{};
      int32_t x[NE], nd_, ns_;
      load_entries(u, nu, x, nd_, ns_);
      if (!__all_sync(0xffffffffu, mbar_wait_idle(dempty, (di & 1) ^ 1))) { okq = false; break; }
      if (lane == 0) {
        desc[0] = u < num_units;
        desc[1] = nu.b;
        desc[2] = nu.g;
        desc[3] = nu.part;
        desc[4] = nu.t0;
        desc[5] = nu.t1;
        desc[6] = nu.nchunks;
        desc[7] = nu.hg;
        desc[8] = nu.single;
        desc[9] = nu.pack;
        desc[10] = nd_;
        desc[11] = ns_;
      }
#pragma unroll
      for (int k = 0; k < NE; ++k) desc[L::kDescHead + 32 * k + lane] = x[k];
      __syncwarp();
      if (lane == 0) mbar_arrive(dfull);
      ++di;
      if (first) {
        first = false;
        wait_prior_grid();
        allow_next_grid();
      }
      if (u >= num_units) break;
      int raw = 0;
      if (lane == 0) raw = (int)gridDim.x + (int)atomicAdd(sched, 1u);
      u = __shfl_sync(0xffffffffu, raw, 0);
    }
    if (!okq && lane == 0) raise_error(PA_DEVERR_TIMEOUT);
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the units: its lanes load a unit's table entries
    // (at most 512 / 8 = 64) in one go, lane 0 takes them by shuffle and
    // issues the copies.  Waits are polled by every lane and voted.
    if (lane == 0) {
      tc::prefetch_tensormap(&tmap_k);
      tc::prefetch_tensormap(&tmap_v);
      tc::prefetch_tensormap(&tmap_q);
    }
    const uint64_t pol_kv = policy_evict_first();
    const uint64_t pol_q = tc::policy_evict_last();
    const int blocks_per_chunk = L::kChunk / bs;
    const int blocks_per_pack = kPackRows / bs;  // blocks of one head in a packed chunk
    const int oob_group = p.num_blocks * p.Hkv * (bs / 8);  // first 8-row group past the pool
    int c = 0, qi = 0;
    bool ok = true;
    // the next unit's description, as the scheduler warp wrote it
    int di = 0;
    bool valid = false;
    auto take = [&](TcUnit &nu, int32_t (&x)[NE], int32_t &nd_, int32_t &ns_) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(dfull, di & 1))) return false;
      valid = desc[0] != 0;
      nu.b = desc[1];
      nu.g = desc[2];
      nu.part = desc[3];
      nu.t0 = desc[4];
      nu.t1 = desc[5];
      nu.nchunks = desc[6];
      nu.hg = desc[7];
      nu.single = desc[8] != 0;
      nu.pack = desc[9] != 0;
      nd_ = desc[10];
      ns_ = desc[11];
#pragma unroll
      for (int k = 0; k < NE; ++k) x[k] = desc[L::kDescHead + 32 * k + lane];
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty);
      ++di;
      return true;
    };
    TcUnit un{};
    int32_t e[NE], nd, ns;
    int u = blockIdx.x;  // without the scheduler: the first unit of every CTA is fixed, later ones drawn
    if (use_sched) {
      if (!take(un, e, nd, ns)) ok = false;
    } else {
      load_entries(u, un, e, nd, ns);
      valid = u < num_units;
    }
    if (!p.late_wait) wait_prior_grid();  // the copies read the pool and Q, which may be written just before
    allow_next_grid();
    while (ok && valid) {
      const int nb_unit = (un.t1 - un.t0 + bs - 1) >> lg_bs;
      const int hstep = un.pack ? kPackHeads : 1;
      // one (sequence, kv head, partition) at a time, or kPackHeads heads in a packed pass
      for (int hh = 0; hh < un.hg; hh += hstep) {
        const int g = un.g + hh;
        const int qs = qi & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&qempty[qs], ((qi >> 1) & 1) ^ 1))) { ok = false; break; }
        {  // publish the unit to the MMA lane and the softmax warpgroup
          int32_t *us = unit_slots + qs * L::kUnitInts;
          if (lane == 0) {
            us[0] = un.b;
            us[1] = g;
            us[2] = un.part;
            us[3] = un.t0;
            us[4] = un.t1;
            us[5] = un.nchunks;
            us[6] = un.single;
            us[7] = nd;
            us[8] = ns;
            us[9] = un.pack;
          }
#pragma unroll
          for (int k = 0; k < NE; ++k) us[L::kUnitHead + 32 * k + lane] = e[k];
          __syncwarp();
        }
        if (lane == 0) {
          uint8_t *qdst = smem + L::kOffQ + qs * L::kQ;
          const int qy = un.b * p.Hq + g * G;
          mbar_arrive_expect_tx(&qfull[qs], L::kQ);
          tc::tma_load_3d(qdst, &tmap_q, 0, qy, 0, &qfull[qs], pol_q);
        }
        ++qi;
        for (int ci = 0; ci < un.nchunks; ++ci, ++c) {
          const int slot = c % 3, use = c / 3;
          for (int which = 0; which < 2; ++which) {  // 0: K ring, 1: V ring
            uint64_t *empty = which ? &vempty[slot] : &kempty[slot];
            uint64_t *full = which ? &vfull[slot] : &kfull[slot];
            const CUtensorMap *map = which ? &tmap_v : &tmap_k;
            if (!__all_sync(0xffffffffu, mbar_wait(empty, (use & 1) ^ 1))) { ok = false; break; }
            uint8_t *dst = smem + (which ? L::kOffV : L::kOffK) + slot * L::kTile;
            if (lane == 0) mbar_arrive_expect_tx(full, L::kTile);
            __syncwarp();
            // lane j loads block j of the chunk (rows j bs ..), or in a packed
            // pass block j % bpp of head j / bpp (bpp blocks per head); a
            // chunk's entries lie in one 32-entry group (blocks_per_chunk and
            // blocks_per_pack divide 32)
            const int bpc = un.pack ? blocks_per_pack : blocks_per_chunk;
            const int jloc = ci * bpc + (lane % bpc);
            const int head = g + (un.pack ? (lane / bpc) % kPackHeads : 0);
            const int32_t blk = __shfl_sync(0xffffffffu, pick(e, (ci * bpc) >> 5), jloc & 31);
            if (lane < blocks_per_chunk) {
              int w = oob_group;
              if (jloc < nb_unit) {
                if (blk >= 0 && blk < p.num_blocks) w = (blk * p.Hkv + head) * (bs / 8);
                else if (which == 0 && hh == 0) raise_error(PA_DEVERR_TABLE);
              }
              tc::tma_load_4d(dst + lane * (bs / 8) * L::kGroup, map, 0, 0, 0, w, full, pol_kv);
            }
          }
          if (!ok) break;
        }
        if (!ok) break;
      }
      if (!ok) break;
      if (use_sched) {
        // the next unit, which the scheduler warp drew and looked up while
        // this one's copies went out
        if (!take(un, e, nd, ns)) { ok = false; break; }
      } else {
        // The next unit is drawn only now, with the ring full of this unit's
        // chunks (which hide the draw's latency): a CTA never holds more work
        // than that when the queue runs dry, so all CTAs finish together.
        // The copy on write goes out while the draw is in flight.
        int raw_next = 0;
        if (lane == 0) raw_next = (int)gridDim.x + (int)atomicAdd(sched, 1u);
        u = __shfl_sync(0xffffffffu, raw_next, 0);
        load_entries(u, un, e, nd, ns);
        valid = u < num_units;
      }
    }
    if (ok) {  // no work left: publish an empty unit so the consumers stop
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
      // wait (bounded) for the copies that may still be in flight
      for (int k = (c > 3 ? c - 3 : 0); k <= c; ++k) {
        mbar_wait(&kfull[k % 3], (k / 3) & 1, 100000000ull);
        mbar_wait(&vfull[k % 3], (k / 3) & 1, 100000000ull);
      }
      for (int k = (qi > 2 ? qi - 2 : 0); k < qi; ++k) mbar_wait(&qfull[k & 1], (k >> 1) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Lane 0 issues the MMAs and their commits; the whole warp polls the
    // waits (voted).  In a fused step the lanes also write the newest token's
    // key row (lanes 0-15, 16 bytes each, once the K tile has landed, before
    // the QK MMA) and value row (lanes 16-31, once the V tile has landed,
    // before the PV MMA) into the tiles of its chunk, and store them to the
    // pool.
    if (!p.late_wait) wait_prior_grid();
    allow_next_grid();
    constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(128, N, false, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(128, N, true, false);
    const uint32_t kbase0 = smem_u32(smem + L::kOffK), vbase0 = smem_u32(smem + L::kOffV);
    const uint32_t qbase0 = smem_u32(smem + L::kOffQ), pbase0 = smem_u32(smem + L::kOffP);
    bool ok = true;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    // smem offset of the 16-byte piece `piece` of column half `half` of row
    // r in a K or V tile: 8-row group r / 8, half at +1 KiB, row r % 8 of
    // the 1 KiB swizzle atom, piece j at position j ^ (r % 8)
    auto tile_piece = [](int r, int half, int piece) {
      return (r >> 3) * L::kGroup + half * 1024 + (r & 7) * 128 + ((piece ^ (r & 7)) << 4);
    };
    // A packed pass has one newest token per head: rows patch + j kPackRows
    // (j < npatch) of the chunk.
    constexpr int kNP = kCanPack ? kPackHeads : 1;
    struct PvJob {
      int c;       // chunk
      int u;       // unit (its O accumulator is u & 1)
      bool first;  // first chunk of the unit: the PV starts the accumulator
      int patch;   // row of the newest token in this chunk, or -1
      int npatch;  // heads with a newest-token row in it
      uint4 vrow[kNP];  // lanes 16-31: their 16 bytes of each value row
      uint4 *pool[kNP]; // lanes 16-31: where those go in the pool
    };
    auto issue_pv = [&](const PvJob &j) -> bool {
      const int c = j.c;
      if (!warp_wait(&pfull[c & 1], (c >> 1) & 1)) return false;
      if (!warp_wait(&vfull[c % 3], (c / 3) & 1)) return false;
      // the accumulator is free once the epilogue of the unit two back read it
      if (j.first && !warp_wait(&ofree[j.u & 1], ((j.u >> 1) & 1) ^ 1)) return false;
      if (j.patch >= 0) {
        if (lane >= 16) {
#pragma unroll
          for (int h = 0; h < kNP; ++h) {
            if (h < j.npatch) {
              const int off = tile_piece(j.patch + h * kPackRows, (lane >> 3) & 1, lane & 7);
              *reinterpret_cast<uint4 *>(smem + L::kOffV + (c % 3) * L::kTile + off) = j.vrow[h];
              *j.pool[h] = j.vrow[h];
            }
          }
          fence_proxy_async_smem();  // before the PV MMA reads the tile
        }
        __syncwarp();
      }
      if (lane == 0) {
        tc::fence_after_sync();
        const uint32_t vb = vbase0 + (c % 3) * L::kTile;
        const uint32_t pb = pbase0 + (c & 1) * L::kP;
        const uint32_t d = tmem + 2 * N + (j.u & 1) * N;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // V^T, MN-major: M = head dim (two 64-wide atoms 1 KiB apart), K = 16
          // tokens = two 8-row groups L::kGroup apart
          const uint64_t a = tc::smem_desc_sw128(vb + kk * 2 * L::kGroup, 1024, L::kGroup);
          const uint64_t bdesc = tc::smem_desc_sw128(pb + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(d, a, bdesc, idesc_pv, (kk > 0 || !j.first) ? 1u : 0u);
        }
        tc::mma_commit(&pvdone[c & 1]);
        tc::mma_commit(&vempty[c % 3]);
      }
      __syncwarp();
      return true;
    };
    int c = 0, qi = 0;
    PvJob pending{};
    pending.c = -1;
    pending.patch = -1;
    while (ok) {
      const int qs = qi & 1;
      if (!warp_wait(&qfull[qs], (qi >> 1) & 1)) { ok = false; break; }
      const int32_t *us = unit_slots + qs * L::kUnitInts;
      const int nchunks = us[5];
      if (nchunks == 0) break;  // the producer ran out of work
      // fused step: this unit's newest token, its chunk and row there, and
      // the lane's 16 bytes of its key (lanes 0-15) or value (16-31) row
      const int32_t nd = us[7];
      const bool upack = us[9] != 0;
      int patch_chunk = -1, patch_row = 0;
      const int npatch = upack ? kPackHeads : 1;
      uint4 nrow[kNP];
      uint4 *pool_row[kNP];
#pragma unroll
      for (int h = 0; h < kNP; ++h) {
        nrow[h] = make_uint4(0, 0, 0, 0);
        pool_row[h] = nullptr;
      }
      if (nd >= 0) {
        const int b = us[0], g = us[1], t0 = us[3], t1 = us[4];
        const int rows = upack ? kPackRows : L::kChunk;  // tokens of one head in a chunk
        patch_chunk = (t1 - 1 - t0) / rows;
        patch_row = (t1 - 1 - t0) % rows;
#pragma unroll
        for (int h = 0; h < kNP; ++h) {
          if (h < npatch) {
            const uint4 *src = static_cast<const uint4 *>(lane < 16 ? p.k_new : p.v_new) +
                               ((size_t)b * p.Hkv + g + h) * 16 + (lane & 15);
            nrow[h] = *src;
            pool_row[h] = static_cast<uint4 *>(const_cast<void *>(lane < 16 ? p.k : p.v)) +
                          (((size_t)nd * p.Hkv + g + h) * p.bs + (t1 - 1) % p.bs) * 16 + (lane & 15);
          }
        }
      }
      const uint32_t qb = qbase0 + qs * L::kQ;
      for (int ci = 0; ci < nchunks; ++ci, ++c) {
        const int slot = c % 3;
        if (!warp_wait(&kfull[slot], (c / 3) & 1)) { ok = false; break; }
        if (ci == patch_chunk) {
          if (lane < 16) {
#pragma unroll
            for (int h = 0; h < kNP; ++h) {
              if (h < npatch) {
                const int off = tile_piece(patch_row + h * kPackRows, (lane >> 3) & 1, lane & 7);
                *reinterpret_cast<uint4 *>(smem + L::kOffK + slot * L::kTile + off) = nrow[h];
                *pool_row[h] = nrow[h];
              }
            }
            fence_proxy_async_smem();  // before the QK MMA reads the tile
          }
          __syncwarp();
        }
        if (lane == 0) {
          tc::fence_after_sync();
          const uint32_t kb = kbase0 + slot * L::kTile;
          const uint32_t d = tmem + (c & 1) * N;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K, K-major: 8-row groups L::kGroup apart, column half kk/4 at +1 KiB
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
        if (pending.c >= 0 && !issue_pv(pending)) { ok = false; break; }
        pending.c = c;
        pending.u = qi;
        pending.first = ci == 0;
        pending.patch = ci == patch_chunk ? patch_row : -1;
        pending.npatch = npatch;
#pragma unroll
        for (int h = 0; h < kNP; ++h) {
          pending.vrow[h] = nrow[h];
          pending.pool[h] = pool_row[h];
        }
      }
      ++qi;
    }
    if (ok && pending.c >= 0 && !issue_pv(pending)) ok = false;
    if (!ok && lane == 0) raise_error(PA_DEVERR_TIMEOUT);
    // no MMA may still be running when the CTA frees its tensor memory
    if (lane == 0) tc::mma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0);
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax + epilogue
    if (!p.late_wait) wait_prior_grid();  // before the first write of out / the workspace
    allow_next_grid();
    const int wq = warp & 3;              // this warp's quarter of the TMEM lanes
    const int r = wq * 32 + lane;         // token row (softmax) / head-dim row (O)
    if (blockIdx.x == 0) {  // rows no unit writes (empty or invalid length): zeros
      for (int b = r; b < p.B; b += 128) {
        const int ctx = COARSE ? p.lens[b] : ctx_s[b];
        if (ctx <= 0 || ctx > p.max_ctx) {
          uint4 *o = reinterpret_cast<uint4 *>(out + (size_t)b * p.Hq * 128);
          for (int e = 0; e < p.Hq * 128 / 8; ++e) o[e] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const int bs = p.bs;
    float m[G], l[G], m_done[G], l_done[G];
#pragma unroll
    for (int n = 0; n < G; ++n) {
      m[n] = -INFINITY;
      l[n] = 0.f;
      m_done[n] = -INFINITY;
      l_done[n] = 0.f;
    }
    TcUnit pun{};        // the unit whose epilogue is pending
    bool pend = false;
    int p_clast = 0;     // its last chunk
    int p_u = 0;         // its index (O accumulator p_u & 1)
    bool bad = false;    // this warp gave up on a wait (warp-uniform)
    bool stop = false;   // some warp of the warpgroup did (uniform: from wg_sync_or)

    // Waits are voted across the warp so that `bad` stays warp-uniform: the
    // tensor-memory loads and stores after them are warp-collective.
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      if (!bad && !__all_sync(0xffffffffu, mbar_wait(bar, parity))) bad = true;
    };

    // O of unit pun (complete once the PV of its last chunk is) and the
    // warpgroup-wide sums l -> the output row, or the partition's statistics.
    // A head-packed pass: each warp's sums and maxima are its own head's
    // (columns wq G ..), all 4 G columns go out.
    auto epilogue_packed = [&]() {
      float o[16];
      warp_wait(&pvdone[p_clast & 1], (p_clast >> 1) & 1);
      if (!bad) {
        tc::fence_after_sync();
        tc::tmem_ld16(trow + 2 * N + (p_u & 1) * N, o);
      }
      tc::fence_before_sync();
      mbar_arrive(&ofree[p_u & 1]);
      const int parity = p_u & 1;
      {
        float v[G];
        float md = 0.f;
#pragma unroll
        for (int n = 0; n < G; ++n) {
          v[n] = l_done[n];
          if (lane == n) md = m_done[n];
        }
        const float t = warp_reduce_columns<G, false>(v, lane);
        if (lane < G) {
          red_sum[(parity * 4 + wq) * N + lane] = t;
          pk_mdone[parity * N + wq * G + lane] = md;
        }
      }
      stop = wg_sync_or(bad);
      if (stop) return;
      constexpr int NC = kPackHeads * G < 16 ? kPackHeads * G : 16;  // the pass's columns
      float Ls[NC];
#pragma unroll
      for (int n = 0; n < NC; ++n) Ls[n] = red_sum[(parity * 4 + n / G) * N + n % G];
      const size_t hrow = (size_t)pun.b * p.Hq + pun.g * G;  // query row of head 0 of the pass
      if (pun.single) {
        __nv_bfloat16 *dst = out + hrow * 128 + r;
#pragma unroll
        for (int n = 0; n < NC; ++n) dst[(size_t)n * 128] = __float2bfloat16_rn(Ls[n] > 0.f ? o[n] / Ls[n] : 0.f);
      } else {
        const size_t row0 = hrow * p.row_stride + pun.part, rs = p.row_stride;
        float *acc = p.ws_acc + row0 * 128 + r;
#pragma unroll
        for (int n = 0; n < NC; ++n) acc[n * rs * 128] = o[n];
        if (r == 0) {
#pragma unroll
          for (int n = 0; n < NC; ++n) {
            p.ws_m[row0 + n * rs] = pk_mdone[parity * N + n];
            p.ws_l[row0 + n * rs] = Ls[n];
          }
        }
      }
    };
    auto epilogue = [&]() {
      if (kCanPack && pun.pack) {
        epilogue_packed();
        return;
      }
      float o[8];
      warp_wait(&pvdone[p_clast & 1], (p_clast >> 1) & 1);
      if (!bad) {
        tc::fence_after_sync();
        tc::tmem_ld8(trow + 2 * N + (p_u & 1) * N, o);
      }
      tc::fence_before_sync();
      mbar_arrive(&ofree[p_u & 1]);
      const int parity = p_u & 1;
      {  // this warp's part of every head's sum; lane n holds head n % G
        float v[G];
#pragma unroll
        for (int n = 0; n < G; ++n) v[n] = l_done[n];
        const float t = warp_reduce_columns<G, false>(v, lane);
        if (lane < G) red_sum[(parity * 4 + wq) * N + lane] = t;
      }
      stop = wg_sync_or(bad);
      if (stop) return;
      float Ls[G];
      combine_warps<G, false>(red_sum + parity * 4 * N, N, 0.f, Ls);
      const size_t hrow = (size_t)pun.b * p.Hq + pun.g * G;  // query row of head 0 of the group
      if (pun.single) {
        __nv_bfloat16 *dst = out + hrow * 128 + r;
#pragma unroll
        for (int n = 0; n < G; ++n) dst[(size_t)n * 128] = __float2bfloat16_rn(Ls[n] > 0.f ? o[n] / Ls[n] : 0.f);
      } else {
        const size_t row0 = hrow * p.row_stride + pun.part, rs = p.row_stride;
        float *acc = p.ws_acc + row0 * 128 + r;
#pragma unroll
        for (int n = 0; n < G; ++n) acc[n * rs * 128] = o[n];
        if (r == 0) {
#pragma unroll
          for (int n = 0; n < G; ++n) {
            p.ws_m[row0 + n * rs] = m_done[n];
            p.ws_l[row0 + n * rs] = Ls[n];
          }
        }
      }
    };

    const int log2_bs = bs == 8 ? 3 : (bs == 16 ? 4 : 5);
    uint32_t p_plain = 0;  // bit i: the last chunk to write P buffer i was a plain one
    int c = 0, qi = 0;
    for (; !stop; ++qi) {
      // the unit, as the producer published it with its Q tile
      const int qs = qi & 1;
      warp_wait(&qfull[qs], (qi >> 1) & 1);
      stop = wg_sync_or(bad);  // every thread reads the slot, or none does
      if (stop) break;
      const int32_t *us = unit_slots + qs * L::kUnitInts;
      TcUnit un;
      un.b = us[0];
      un.g = us[1];
      un.part = us[2];
      un.t0 = us[3];
      un.t1 = us[4];
      un.nchunks = us[5];
      un.single = us[6] != 0;
      un.pack = kCanPack && us[9] != 0;
      if (un.nchunks == 0) break;  // the producer ran out of work
      const int32_t *ents = us + L::kUnitHead;
      const int tail_end = min(((un.t1 + bs - 1) >> log2_bs) << log2_bs, un.t0 + PART);
      const uint32_t obuf = trow + 2 * N + (qi & 1) * N;
      // Copy on write of the unit's newest block (fused step): the source
      // tile over the destination's, every row but the new one (the MMA warp
      // stores that).  Nothing in this call reads the destination.  Thread r
      // takes vectors r, r + 128, ... of the K and V tiles; the first two are
      // loaded now and stored once the first chunk's weights are out.
      const int32_t cw_src = us[8], cw_dst = us[7];
      const int cw_vecs = bs * 16, cw_skip = (un.t1 - 1) & (bs - 1);
      uint4 cwk[2], cwv[2];
      if (cw_src >= 0) {
        const size_t s0 = ((size_t)cw_src * p.Hkv + un.g) * cw_vecs;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = r + 128 * j;
          if (i < cw_vecs) {
            cwk[j] = static_cast<const uint4 *>(p.k)[s0 + i];
            cwv[j] = static_cast<const uint4 *>(p.v)[s0 + i];
          }
        }
      }
      auto cw_store = [&]() {
        const size_t s0 = ((size_t)cw_src * p.Hkv + un.g) * cw_vecs;
        const size_t d0 = ((size_t)cw_dst * p.Hkv + un.g) * cw_vecs;
        uint4 *kd = static_cast<uint4 *>(const_cast<void *>(p.k)) + d0;
        uint4 *vd = static_cast<uint4 *>(const_cast<void *>(p.v)) + d0;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = r + 128 * j;
          if (i < cw_vecs && (i >> 4) != cw_skip) {
            kd[i] = cwk[j];
            vd[i] = cwv[j];
          }
        }
        for (int i = r + 256; i < cw_vecs; i += 128) {  // 32-token blocks: the rest
          if ((i >> 4) != cw_skip) {
            kd[i] = static_cast<const uint4 *>(p.k)[s0 + i];
            vd[i] = static_cast<const uint4 *>(p.v)[s0 + i];
          }
        }
        if (un.pack) {  // the pass's other heads
          for (int h = 1; h < kPackHeads; ++h) {
            const size_t hs = s0 + (size_t)h * cw_vecs, hd = (size_t)h * cw_vecs;
            for (int i = r; i < cw_vecs; i += 128) {
              if ((i >> 4) != cw_skip) {
                kd[hd + i] = static_cast<const uint4 *>(p.k)[hs + i];
                vd[hd + i] = static_cast<const uint4 *>(p.v)[hs + i];
              }
            }
          }
        }
      };
#pragma unroll
      for (int n = 0; n < G; ++n) {
        m_done[n] = m[n];
        l_done[n] = l[n];
        m[n] = -INFINITY;
        l[n] = 0.f;
      }
      for (int ci = 0; ci < un.nchunks; ++ci, ++c) {
        float s[8];
        warp_wait(&sfull[c & 1], (c >> 1) & 1);
        // packed: this warp's rows are head wq's, its columns wq G ..
        const int col0 = un.pack ? wq * G : 0;
        if (!bad) {
          tc::fence_after_sync();
          tc::tmem_ld8(trow + (c & 1) * N + col0, s);
        }
        const int tok = un.pack ? un.t0 + ci * kPackRows + lane : un.t0 + ci * L::kChunk + r;
        const int32_t blk = tok < un.t1 ? ents[(tok - un.t0) >> log2_bs] : -1;
        const bool valid = blk >= 0 && blk < p.num_blocks;
        // Scores are weighed against the running reference m as long as no
        // score exceeds it by more than kLazyRescale (weights stay below
        // 2^8); only then, warpgroup-wide, is the chunk's exact max taken.
        // The result is the same: the softmax does not depend on the
        // reference.
        float x[G];
        bool need = false;
#pragma unroll
        for (int n = 0; n < G; ++n) {
          x[n] = (valid && !bad) ? s[n] * p.scale_log2 : -INFINITY;
          need |= x[n] > m[n] + kLazyRescale;
        }
        // a masked row inside the partition's last, partly filled block holds
        // whatever the pool has there: zero its V row before PV reads it
        const bool tail_row = tok >= un.t1 && tok < tail_end;
        if (__any_sync(0xffffffffu, tail_row)) {
          warp_wait(&vfull[c % 3], (c / 3) & 1);
          if (!bad && tail_row) {
            uint4 *vr = reinterpret_cast<uint4 *>(smem + L::kOffV + (c % 3) * L::kTile +
                                                  (r >> 3) * L::kGroup + (r & 7) * 128);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              vr[e] = make_uint4(0, 0, 0, 0);
              vr[1024 / 16 + e] = make_uint4(0, 0, 0, 0);
            }
          }
        }
        float mnew[G];
        const bool red_path = wg_sync_or(need || bad);
        if (red_path) {  // uniform: some row needs a new reference (or gave up)
          {  // this warp's max of every head; lane n holds head n % G
            float v[G];
#pragma unroll
            for (int n = 0; n < G; ++n) v[n] = x[n];
            const float t = warp_reduce_columns<G, true>(v, lane);
            if (lane < G) red_max[((c & 1) * 4 + wq) * N + lane] = t;
          }
          stop = wg_sync_or(bad);
          if (stop) break;
          float cm[G];
          if (un.pack) {  // the warp's own head
#pragma unroll
            for (int n = 0; n < G; ++n) cm[n] = red_max[((c & 1) * 4 + wq) * N + n];
          } else {
            combine_warps<G, true>(red_max + (c & 1) * 4 * N, N, -INFINITY, cm);
          }
#pragma unroll
          for (int n = 0; n < G; ++n) mnew[n] = fmaxf(m[n], cm[n]);
        } else {
#pragma unroll
          for (int n = 0; n < G; ++n) mnew[n] = m[n];
        }
        float alpha[G];
        bool moved = false;  // uniform: m and mnew are the same in every thread (packed: in the warp)
#pragma unroll
        for (int n = 0; n < G; ++n) {
          moved |= mnew[n] != m[n];
          alpha[n] = (mnew[n] == m[n]) ? 1.f : ex2_approx(m[n] - mnew[n]);
        }
        if (un.pack && red_path) {
          // every thread rescales all heads' columns of its O row: publish
          // this warp's weights, and agree on whether any head moved
          float a = 1.f;
#pragma unroll
          for (int n = 0; n < G; ++n)
            if (lane == n) a = alpha[n];
          if (lane < G) pk_alpha[(c & 1) * N + wq * G + lane] = a;
          moved = wg_sync_or(moved);
        }
        if (moved && ci > 0) {
          // O of this unit holds the chunks before c weighed against the old
          // reference: rescale it once PV(c-1) has landed, before PV(c) adds
          warp_wait(&pvdone[(c - 1) & 1], ((c - 1) >> 1) & 1);
          if (!bad) {
            tc::fence_after_sync();
            if (kCanPack && un.pack) {
              float o[16];
              tc::tmem_ld16(obuf, o);
#pragma unroll
              for (int n = 0; n < 16; ++n)
                if (n < kPackHeads * G) o[n] *= pk_alpha[(c & 1) * N + n];
              tc::tmem_st16(obuf, o);
            } else {
              float o[8];
              tc::tmem_ld8(obuf, o);
#pragma unroll
              for (int n = 0; n < G; ++n) o[n] *= alpha[n];
              tc::tmem_st8(obuf, o);
            }
          }
        }
        __nv_bfloat16 *pb = reinterpret_cast<__nv_bfloat16 *>(smem + L::kOffP + (c & 1) * L::kP);
        const int kh = r >> 6, rr = r & 63;
        // P^T row n (K-major, 128-byte swizzle): token r in half kh
        auto p_off = [&](int n) {
          return kh * (N * 64) + (n >> 3) * 512 + (n & 7) * 64 + (((rr >> 3) ^ (n & 7)) << 3) + (rr & 7);
        };
#pragma unroll
        for (int n = 0; n < G; ++n) {
          const float pv = valid ? ex2_approx(x[n] - mnew[n]) : 0.f;
          l[n] = fmaf(l[n], alpha[n], pv);
          m[n] = mnew[n];
          pb[p_off(col0 + n)] = __float2bfloat16_rn(pv);
        }
        // A packed chunk needs 0 in the other heads' columns of this row.  A
        // thread's rows are always its warp's head in packed chunks, so those
        // columns stay 0 from its last packed chunk in this buffer; only a
        // plain chunk there since (which writes columns 0 .. G - 1 of every
        // row) makes columns 0 .. G - 1 of the rows of heads 1.. stale.
        if (kCanPack) {
          const uint32_t bit = 1u << (c & 1);
          if (un.pack) {
            if (p_plain & bit) {
              if (wq != 0) {
#pragma unroll
                for (int n = 0; n < G; ++n) pb[p_off(n)] = __float2bfloat16_rn(0.f);
              }
              p_plain &= ~bit;
            }
          } else {
            p_plain |= bit;
          }
        }
        fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(&pfull[c & 1]);
        if (ci == un.nchunks - 1 && threadIdx.x == 64) mbar_arrive(&qempty[qs]);  // done with the unit slot
        // the previous unit's output, while this chunk's PV runs
        if (ci == 0 && pend) {
          epilogue();
          pend = false;
          if (stop) break;
        }
        if (ci == 0 && cw_src >= 0) cw_store();
      }
      if (stop) break;
      pend = true;
      pun = un;
      p_clast = c - 1;
      p_u = qi;
    }
    if (pend && !stop) {
#pragma unroll
      for (int n = 0; n < G; ++n) {
        m_done[n] = m[n];
        l_done[n] = l[n];
      }
      epilogue();
    }
    if (stop) raise_error(PA_DEVERR_TIMEOUT);
  }

  if (p.late_wait) wait_prior_grid();  // complete only after the cascade kernel
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0) {  // this CTA draws no more units; the last one out resets the slot
    __threadfence();
    if (atomicAdd(&sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&sched[0], 0u);
      atomicExch(&sched[1], 0u);
    }
  }
  if (warp == 1) tc::tmem_dealloc(tmem, L::kTmemCols);
}

}  // namespace pa

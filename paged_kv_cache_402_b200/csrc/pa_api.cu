// C ABI of the paged KV-cache path: argument checks, launch configuration and
// the device error word.  Every kernel of the library is compiled in this one
// translation unit (the error word is one __device__ symbol).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <utility>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "pa_copy_kernels.cuh"
#include "pa_decode_simt.cuh"
#include "pa_decode_shared.cuh"
#include "pa_prefill_tc.cuh"
#include "pa_decode_tc.cuh"
#include "pagedattn.h"

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int elem_bytes(int32_t dtype) { return dtype == PA_DTYPE_F32 ? 4 : 2; }

pa_status check_cache(const pa_cache_t *c) {
  if (!c || !c->k || !c->v) return PA_ERR_INVALID_ARG;
  if (c->dtype != PA_DTYPE_F32 && c->dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
  if (c->num_blocks <= 0 || c->num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
  if (c->block_size != 8 && c->block_size != 16 && c->block_size != 32) return PA_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (!aligned16(c->k) || !aligned16(c->v)) return PA_ERR_INVALID_ARG;
  if (c->partition_tokens != 0 && c->partition_tokens != 256 && c->partition_tokens != 512 &&
      c->partition_tokens != 1024)
    return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

// Tokens per split-context partition of decode calls over the pool.
inline int32_t part_of(const pa_cache_t *c) { return c->partition_tokens ? c->partition_tokens : pa::kPart; }

inline bool part_ok(int32_t part) { return part == 256 || part == 512 || part == 1024; }

// The CUDA error behind this thread's most recent PA_ERR_CUDA (0: none).
thread_local int32_t g_last_cuda_error = 0;

inline pa_status cuda_failed(cudaError_t e) {
  g_last_cuda_error = (int32_t)e;
  return PA_ERR_CUDA;
}

inline pa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

// Launches with programmatic stream serialization: the kernel may be
// scheduled while the previous kernel in the stream is finishing; each of
// the library's kernels waits (griddepcontrol.wait) before reading memory.
template <typename... KArgs, typename... Args>
pa_status launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                 Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return cuda_failed(e);
  }
  return launch_status();
}

inline int32_t max_parts_for(int32_t max_context_len, int32_t part) {
  // in 64 bits: a length near INT32_MAX must not wrap before the division
  return (int32_t)(((int64_t)max_context_len + part - 1) / part);
}

inline size_t round16(size_t x) { return (x + 15) & ~(size_t)15; }

constexpr int kMaxDev = 64;

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return -1;
  return dev;
}

// SM count of the current device, looked up once per device.
int sm_count() {
  static std::atomic<int> cache[kMaxDev] = {};
  const int dev = current_device();
  if (dev < 0) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Raises a kernel's dynamic shared-memory limit once per device (and again
// only if a larger size is asked for).  `done` belongs to that one kernel.
template <typename Kernel>
bool ensure_smem(Kernel kern, int bytes, std::atomic<int> (&done)[kMaxDev]) {
  const int dev = current_device();
  if (dev < 0) return false;
  if (done[dev].load(std::memory_order_relaxed) >= bytes) return true;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    g_last_cuda_error = (int32_t)e;
    return false;
  }
  done[dev].store(bytes, std::memory_order_relaxed);
  return true;
}


// workspace layout: m [B*Hq*R] f32 | l [B*Hq*R] f32 | acc [B*Hq*R*D] f32,
// R rows per (sequence, query head): one per partition, plus, with a
// sharing plan (extra), the row of the cascade's piece of the partition a
// shared prefix ends in.
int64_t row_stride_for(int32_t max_ctx, int32_t part, bool extra) {
  return (max_ctx > 0 ? (int64_t)max_parts_for(max_ctx, part) : 1) + (extra ? 1 : 0);
}

size_t workspace_bytes_for(int64_t B, int64_t Hq, int32_t max_ctx, int64_t D, int32_t part,
                           bool extra = false) {
  if (!extra && max_ctx <= part) return 0;
  const int64_t rows = B * Hq * row_stride_for(max_ctx, part, extra);
  return round16(rows * 4) * 2 + round16(rows * D * 4);
}

// Shared-memory ring of the partition kernel: per warp `nstages` slots of a
// K tile and a V tile, then the mbarriers.  Aimed at two CTAs per SM (about
// 24 KiB per warp), at least one slot, never past 192 KiB per CTA.
int choose_stages(int tile_bytes) {
  const int per_warp_budget = 24 * 1024;
  int n = per_warp_budget / (2 * tile_bytes);
  if (n < 2) n = 2;
  if (n > 8) n = 8;
  while (n > 1 && (size_t)pa::kWarps * n * 2 * tile_bytes > 192 * 1024) --n;
  return n;
}

// The partition merge after a decode launch: with at most kReduceWide
// workspace rows per (sequence, query head), a warp-per-row kernel (sized to
// the bound, NP 4, 8 or 16, or the one that reads up to 32 rows in rounds),
// over a grid of at most 4 CTAs per SM; else one CTA per row.
template <typename T, int D>
pa_status launch_reduce(const pa::DecodeParams &p, cudaStream_t st) {
  const int32_t max_parts = p.row_stride;  // rows a merge may read
  if (max_parts > pa::kReduceWide)
    return launch(pa::decode_reduce<T, D>, dim3(p.B * p.Hq), dim3(128), (size_t)max_parts * sizeof(float), st, p);
  const int64_t rows = (int64_t)p.B * p.Hq;
  int64_t grid = (rows + pa::kReduceRowWarps - 1) / pa::kReduceRowWarps;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  if (grid > 4 * (int64_t)sms) grid = 4 * (int64_t)sms;
  const dim3 block(pa::kReduceRowWarps * 32);
  if (max_parts <= 4) return launch(pa::decode_reduce_rows<T, D, 4>, dim3((unsigned)grid), block, 0, st, p);
  if (max_parts <= 8) return launch(pa::decode_reduce_rows<T, D, 8>, dim3((unsigned)grid), block, 0, st, p);
  if (max_parts <= 16) return launch(pa::decode_reduce_rows<T, D, 16>, dim3((unsigned)grid), block, 0, st, p);
  return launch(pa::decode_reduce_rows_wide<T, D>, dim3((unsigned)grid), block, 0, st, p);
}

template <typename T, int D, int G>
pa_status launch_decode_t(const pa::DecodeParams &p, int32_t max_parts, cudaStream_t st) {
  const int tile_bytes = p.bs * D * (int)sizeof(T);
  const int nstages = choose_stages(tile_bytes);
  size_t smem = (size_t)pa::kWarps * nstages * 2 * tile_bytes + (size_t)pa::kWarps * nstages * 8;
  const size_t merge = (size_t)pa::kWarps * G * (D + 2) * sizeof(float);
  if (smem < merge) smem = merge;
  auto kern = pa::decode_partition_simt<T, D, G>;
  static std::atomic<int> smem_set[kMaxDev] = {};
  if (!ensure_smem(kern, (int)smem, smem_set)) return PA_ERR_CUDA;
  dim3 grid(max_parts, p.Hkv, p.B);
  pa_status s = launch(kern, grid, dim3(pa::kWarps * 32), smem, st, p, nstages);
  if (s != PA_OK || max_parts <= 1) return s;
  return launch_reduce<T, D>(p, st);
}

template <typename T, int D>
pa_status launch_decode_d(const pa::DecodeParams &p, int32_t max_parts, cudaStream_t st) {
  switch (p.G) {
    case 1: return launch_decode_t<T, D, 1>(p, max_parts, st);
    case 2: return launch_decode_t<T, D, 2>(p, max_parts, st);
    case 4: return launch_decode_t<T, D, 4>(p, max_parts, st);
    case 8: return launch_decode_t<T, D, 8>(p, max_parts, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------
// tensor-core decode (bf16, head_dim 128, group size <= 8)

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// A [rows][128] bf16 matrix read in boxes of 64 columns x box_rows rows with
// 128-byte swizzle (the layout the MMA descriptors expect).
bool make_map_bf16_d128(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128 * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The paged pool [rows][128] bf16 seen as 4-D (64 columns, 8 rows, 2 column
// halves, 8-row groups) so that one box of (64, 8, 2, bs/8) is a whole
// (block, kv head) tile and lands as [group][half][8 rows x 128 B] with
// 128-byte swizzle.
bool make_map_pool_4d(CUtensorMap *m, const void *base, uint64_t rows, uint32_t bs) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn || rows % 8 || bs % 8) return false;
  const cuuint64_t dims[4] = {64, 8, 2, rows / 8};
  const cuuint64_t strides[3] = {256, 128, 2048};
  const cuuint32_t box[4] = {64, 8, 2, bs / 8};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [total][Hq][128] bf16 seen as 3-D (128 columns, Hq heads, total tokens):
// a box (64, G, Mq) is Mq tokens x the G query heads of one kv head, landing
// as 128-byte rows ordered (token, head) with 128-byte swizzle.
bool make_map_q3d(CUtensorMap *m, const void *base, uint64_t total, uint32_t Hq, uint32_t G, uint32_t Mq) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, Hq, total};
  const cuuint64_t strides[2] = {128 * 2, (cuuint64_t)Hq * 128 * 2};
  const cuuint32_t box[3] = {64, G, Mq};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [rows][128] bf16 seen as 3-D (64 columns, rows, 2 column halves) so that
// one box of (64, box_rows, 2) lands as [half][box_rows rows x 128 B] with
// 128-byte swizzle: a query tile's two column halves in one copy.
bool make_map_q_halves(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, rows, 2};
  const cuuint64_t strides[2] = {128 * 2, 64 * 2};
  const cuuint32_t box[3] = {64, box_rows, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_eligible(const pa::DecodeParams &p, int dtype, int D) {
  if (dtype != PA_DTYPE_BF16 || D != 128) return false;
  if (p.G < 1 || p.G > 8 || (p.G & (p.G - 1))) return false;
  if ((int64_t)p.num_blocks * p.Hkv * p.bs >= (int64_t)INT32_MAX) return false;
  if ((int64_t)p.B * p.Hq >= (int64_t)INT32_MAX) return false;
  return true;  // a missing tensor-map encoder then fails the launch loudly (PA_ERR_CUDA)
}

template <int G, int PART, bool COARSE>
pa_status launch_decode_tc_slice(const pa::DecodeParams &p, int32_t max_parts, cudaStream_t st) {
  CUtensorMap mk, mv, mq;
  const uint64_t rows = (uint64_t)p.num_blocks * p.Hkv * p.bs;
  // a query tile: the kN rows from a group's first query row, both halves
  if (!make_map_pool_4d(&mk, p.k, rows, (uint32_t)p.bs) ||
      !make_map_pool_4d(&mv, p.v, rows, (uint32_t)p.bs) ||
      !make_map_q_halves(&mq, p.q, (uint64_t)p.B * p.Hq, (uint32_t)pa::TcLayout::kN))
    return PA_ERR_CUDA;
  auto kern = pa::decode_partition_tc<G, PART, COARSE>;
  const int smem = pa::TcLayout::kBytes;
  static std::atomic<int> smem_set[kMaxDev] = {};
  if (!ensure_smem(kern, smem, smem_set)) return PA_ERR_CUDA;
  const int64_t units_bound = (int64_t)p.Hkv * p.B * max_parts;
  int grid = sm_count();
  if (grid <= 0) return PA_ERR_CUDA;
  if (units_bound < grid) grid = (int)units_bound;
  return launch(kern, dim3(grid), dim3(pa::TcLayout::kThreads), (size_t)smem, st, mk, mv, mq, p);
}

// Sequences are independent: a batch larger than the kernel's per-CTA
// sequence tables (kMaxSeqs sequences, or kCoarse times that in its coarse
// form) runs as consecutive launches over slices of it, and one reduce over
// the whole batch follows the last (each launch completes only after the one
// before it, so the reduce sees every slice's rows).
std::atomic<uint32_t> g_sched_ticket{0};

template <int G, int PART>
pa_status launch_decode_tc_g(const pa::DecodeParams &p, int32_t max_parts, cudaStream_t st) {
  // a slice is at most kCoarse x kMaxSeqs sequences, and, at most kMaxSeqs
  // of them (the packed prefix sums), its full partitions must fit 20 bits
  int slice = p.B > pa::TcLayout::kMaxSeqs ? pa::kCoarse * pa::TcLayout::kMaxSeqs : pa::TcLayout::kMaxSeqs;
  const int by_parts = ((1 << pa::kFullBits) - 1) / (max_parts > 0 ? max_parts : 1);
  if (by_parts < slice) slice = by_parts > 0 ? by_parts : 1;
  for (int b0 = 0; b0 < p.B; b0 += slice) {
    pa::DecodeParams ps = p;
    ps.B = p.B - b0 < slice ? p.B - b0 : slice;
    const size_t rows = (size_t)b0 * p.Hq;  // (sequence, query head) rows before the slice
    ps.q = static_cast<const __nv_bfloat16 *>(p.q) + rows * 128;
    ps.out = static_cast<__nv_bfloat16 *>(p.out) + rows * 128;
    ps.tables = p.tables + (size_t)b0 * p.max_blocks;
    ps.lens = p.lens + b0;
    if (p.k_new) {  // fused step: the slice's new rows and copy sources
      ps.k_new = static_cast<const __nv_bfloat16 *>(p.k_new) + (size_t)b0 * p.Hkv * 128;
      ps.v_new = static_cast<const __nv_bfloat16 *>(p.v_new) + (size_t)b0 * p.Hkv * 128;
      if (p.cow_src) ps.cow_src = p.cow_src + b0;
    }
    if (p.first_tok) ps.first_tok = p.first_tok + b0;
    if (p.ws_m) {
      ps.ws_m = p.ws_m + rows * p.row_stride;
      ps.ws_l = p.ws_l + rows * p.row_stride;
      ps.ws_acc = p.ws_acc + rows * p.row_stride * 128;
    }
    ps.sched_slot = (int32_t)(g_sched_ticket.fetch_add(1) % pa::kSchedSlots);
    const pa_status s = ps.B > pa::TcLayout::kMaxSeqs ? launch_decode_tc_slice<G, PART, true>(ps, max_parts, st)
                                                       : launch_decode_tc_slice<G, PART, false>(ps, max_parts, st);
    if (s != PA_OK) return s;
  }
  if (p.row_stride <= 1) return PA_OK;  // one partition, no plan: written directly
  return launch_reduce<__nv_bfloat16, 128>(p, st);
}

// The cascade kernel over the shared tokens of a sharing plan, in slices of
// at most kMaxGroups groups.
template <int G, int PART>
pa_status launch_decode_shared_g(const pa::DecodeParams &p, const pa_share_plan_t &plan, cudaStream_t st) {
  CUtensorMap mk, mv, mq;
  const uint64_t rows = (uint64_t)p.num_blocks * p.Hkv * p.bs;
  if (!make_map_pool_4d(&mk, p.k, rows, (uint32_t)p.bs) ||
      !make_map_pool_4d(&mv, p.v, rows, (uint32_t)p.bs) ||
      !make_map_bf16_d128(&mq, p.q, (uint64_t)p.B * p.Hq, (uint32_t)G))
    return PA_ERR_CUDA;
  auto kern = pa::decode_shared_tc<G, PART>;
  const int smem = pa::ShLayout::kBytes;
  static std::atomic<int> smem_set[kMaxDev] = {};
  if (!ensure_smem(kern, smem, smem_set)) return PA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  for (int j0 = 0; j0 < plan.n_groups; j0 += pa::ShLayout::kMaxGroups) {
    pa::SharedParams sp{};
    sp.n_groups = plan.n_groups - j0 < pa::ShLayout::kMaxGroups ? plan.n_groups - j0 : pa::ShLayout::kMaxGroups;
    sp.max_members = plan.max_members;
    sp.members = plan.members + (size_t)j0 * plan.max_members;
    sp.shared = plan.shared_tokens + j0;
    const int64_t units_bound = (int64_t)sp.n_groups * p.Hkv * (p.max_parts > 0 ? p.max_parts : 1);
    const int grid = units_bound < sms ? (int)units_bound : sms;
    const pa_status s = launch(kern, dim3(grid), dim3(pa::ShLayout::kThreads), (size_t)smem, st, mk, mv, mq, p, sp);
    if (s != PA_OK) return s;
  }
  return PA_OK;
}

template <int PART>
pa_status launch_decode_shared_p(const pa::DecodeParams &p, const pa_share_plan_t &plan, cudaStream_t st) {
  switch (p.G) {
    case 1: return launch_decode_shared_g<1, PART>(p, plan, st);
    case 2: return launch_decode_shared_g<2, PART>(p, plan, st);
    case 4: return launch_decode_shared_g<4, PART>(p, plan, st);
    case 8: return launch_decode_shared_g<8, PART>(p, plan, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

pa_status launch_decode_shared(const pa::DecodeParams &p, const pa_share_plan_t &plan, cudaStream_t st) {
  switch (p.part) {
    case 256: return launch_decode_shared_p<256>(p, plan, st);
    case 512: return launch_decode_shared_p<512>(p, plan, st);
    case 1024: return launch_decode_shared_p<1024>(p, plan, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

// Chunked prefill, in slices of at most kMaxSeqs sequences.
template <int G>
pa_status launch_prefill_g(const pa::DecodeParams &p, const int32_t *qstart, int64_t total_q,
                           int32_t max_query_len, cudaStream_t st) {
  constexpr int Mq = pa::PfLayout::kM / G;
  CUtensorMap mk, mv, mq;
  const uint64_t rows = (uint64_t)p.num_blocks * p.Hkv * p.bs;
  if (!make_map_pool_4d(&mk, p.k, rows, (uint32_t)p.bs) ||
      !make_map_pool_4d(&mv, p.v, rows, (uint32_t)p.bs) ||
      !make_map_q3d(&mq, p.q, (uint64_t)total_q, (uint32_t)p.Hq, (uint32_t)G, (uint32_t)Mq))
    return PA_ERR_CUDA;
  auto kern = pa::prefill_tc<G>;
  const int smem = pa::PfLayout::kBytes;
  static std::atomic<int> smem_set[kMaxDev] = {};
  if (!ensure_smem(kern, smem, smem_set)) return PA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  for (int b0 = 0; b0 < p.B; b0 += pa::PfLayout::kMaxSeqs) {
    pa::DecodeParams ps = p;
    ps.B = p.B - b0 < pa::PfLayout::kMaxSeqs ? p.B - b0 : pa::PfLayout::kMaxSeqs;
    ps.tables = p.tables + (size_t)b0 * p.max_blocks;
    ps.lens = p.lens + b0;
    ps.sched_slot = (int32_t)(g_sched_ticket.fetch_add(1) % pa::kSchedSlots);
    pa::PrefillParams pp{qstart + b0, Mq};
    const int64_t units_bound = (int64_t)ps.B * p.Hkv * ((max_query_len + Mq - 1) / Mq);
    const int grid = units_bound < sms ? (int)(units_bound > 0 ? units_bound : 1) : sms;
    const pa_status s = launch(kern, dim3(grid), dim3(pa::PfLayout::kThreads), (size_t)smem, st, mk, mv, mq, ps, pp);
    if (s != PA_OK) return s;
  }
  return PA_OK;
}

template <int PART>
pa_status launch_decode_tc_p(const pa::DecodeParams &p, int32_t max_parts, cudaStream_t st) {
  switch (p.G) {
    case 1: return launch_decode_tc_g<1, PART>(p, max_parts, st);
    case 2: return launch_decode_tc_g<2, PART>(p, max_parts, st);
    case 4: return launch_decode_tc_g<4, PART>(p, max_parts, st);
    case 8: return launch_decode_tc_g<8, PART>(p, max_parts, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

pa_status launch_decode_tc(const pa::DecodeParams &p, int32_t max_parts, cudaStream_t st) {
  switch (p.part) {
    case 256: return launch_decode_tc_p<256>(p, max_parts, st);
    case 512: return launch_decode_tc_p<512>(p, max_parts, st);
    case 1024: return launch_decode_tc_p<1024>(p, max_parts, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

template <typename T>
pa_status launch_decode_dtype(const pa::DecodeParams &p, int D, int32_t max_parts,
                              cudaStream_t st) {
  if (D == 64) return launch_decode_d<T, 64>(p, max_parts, st);
  if (D == 128) return launch_decode_d<T, 128>(p, max_parts, st);
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

PA_API const char *pa_version(void) { return "0.1.0"; }

PA_API int32_t pa_last_cuda_error(void) { return g_last_cuda_error; }

PA_API const char *pa_cuda_error_string(int32_t code) {
  return cudaGetErrorString(static_cast<cudaError_t>(code));
}

PA_API const char *pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported dtype, head_dim, block_size or group size";
    case PA_ERR_OUT_OF_BLOCKS: return "out of free blocks";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_NOT_FOUND: return "no such sequence";
    case PA_ERR_TOO_SMALL: return "buffer too small";
  }
  return "unknown status";
}

PA_API pa_status pa_append_kv(const void *k, const void *v, const int64_t *slot_mapping,
                              int32_t num_tokens, const pa_cache_t *cache, void *stream) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !aligned16(k) || !aligned16(v)) return PA_ERR_INVALID_ARG;
  const int row_bytes = cache->head_dim * elem_bytes(cache->dtype);
  const int row_vecs = row_bytes / 16;
  const int64_t warps = (int64_t)num_tokens * cache->num_kv_heads;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > INT32_MAX) return PA_ERR_INVALID_ARG;
  return launch(pa::append_kv_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream,
                (const uint4 *)k, (const uint4 *)v, slot_mapping, num_tokens, cache->num_kv_heads,
                cache->block_size, row_vecs, (int64_t)cache->num_blocks * cache->block_size,
                (uint4 *)cache->k, (uint4 *)cache->v);
}

PA_API pa_status pa_copy_blocks(const int32_t *src_dst_pairs, int32_t num_pairs,
                                const pa_cache_t *cache, void *stream) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (num_pairs < 0 || num_pairs > 65535) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!src_dst_pairs) return PA_ERR_INVALID_ARG;
  const int64_t block_bytes = (int64_t)cache->block_size * cache->num_kv_heads * cache->head_dim *
                              elem_bytes(cache->dtype);
  const int64_t block_vecs = block_bytes / 16;
  const int64_t per_cta = 256 * pa::kCopyUnroll;
  dim3 grid((unsigned)((block_vecs + per_cta - 1) / per_cta), (unsigned)num_pairs);
  return launch(pa::copy_blocks_kernel, grid, dim3(256), 0, (cudaStream_t)stream, src_dst_pairs,
                cache->num_blocks, block_vecs, (uint4 *)cache->k, (uint4 *)cache->v);
}

PA_API pa_status pa_check_copy_pairs(const int32_t *pairs, int32_t num_pairs, int32_t num_blocks) {
  if (num_pairs < 0 || num_blocks <= 0 || (num_pairs > 0 && !pairs)) return PA_ERR_INVALID_ARG;
  std::vector<uint8_t> role(num_blocks, 0);  // bit 0: a source, bit 1: a destination
  for (int32_t i = 0; i < num_pairs; ++i) {
    const int32_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return PA_ERR_INVALID_ARG;
    if (role[dst] & 2) return PA_ERR_INVALID_ARG;  // repeated destination
    role[src] |= 1;
    role[dst] |= 2;
  }
  for (int32_t b = 0; b < num_blocks; ++b)
    if (role[b] == 3) return PA_ERR_INVALID_ARG;  // a destination that is also a source
  return PA_OK;
}

PA_API size_t pa_decode_workspace_size_p(int32_t num_seqs, int32_t num_q_heads,
                                         int32_t max_context_len, int32_t head_dim,
                                         int32_t partition_tokens) {
  const int32_t part = partition_tokens ? partition_tokens : pa::kPart;
  if (num_seqs <= 0 || num_q_heads <= 0 || max_context_len <= 0 || head_dim <= 0 || !part_ok(part)) return 0;
  return workspace_bytes_for(num_seqs, num_q_heads, max_context_len, head_dim, part);
}

PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                       int32_t max_context_len, int32_t head_dim) {
  return pa_decode_workspace_size_p(num_seqs, num_q_heads, max_context_len, head_dim, pa::kPart);
}

PA_API size_t pa_decode_shared_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t max_context_len, int32_t head_dim,
                                              int32_t partition_tokens) {
  const int32_t part = partition_tokens ? partition_tokens : pa::kPart;
  if (num_seqs <= 0 || num_q_heads <= 0 || max_context_len <= 0 || head_dim <= 0 || !part_ok(part)) return 0;
  return workspace_bytes_for(num_seqs, num_q_heads, max_context_len, head_dim, part, true);
}

}  // extern "C"

namespace {

// Checks pa_decode's arguments and fills the kernel parameters.  *skip is
// set when there is nothing to launch (no sequences).
pa_status prepare_decode(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                         int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
                         int32_t num_q_heads, int32_t max_context_len, float scale, void *out,
                         void *workspace, size_t workspace_bytes, pa::DecodeParams *pp,
                         bool *skip, bool extra_row = false) {
  *skip = false;
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0 || max_blocks_per_seq < 0)
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) {
    *skip = true;
    return PA_OK;
  }
  if (!q || !out || !block_tables || !context_lens || !aligned16(q) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int32_t G = num_q_heads / cache->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || cache->num_kv_heads > 65535) return PA_ERR_INVALID_ARG;
  const int32_t bs = cache->block_size;
  if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * bs) return PA_ERR_INVALID_ARG;
  const int32_t part = part_of(cache);
  if (max_context_len > INT32_MAX - part) return PA_ERR_INVALID_ARG;
  const size_t need = workspace_bytes_for(num_seqs, num_q_heads, max_context_len, cache->head_dim, part, extra_row);
  if (need > 0) {
    if (!workspace || !aligned16(workspace)) return PA_ERR_INVALID_ARG;
    if (workspace_bytes < need) return PA_ERR_TOO_SMALL;
  }
  const int32_t max_parts = max_context_len > 0 ? max_parts_for(max_context_len, part) : 1;
  const int64_t row_stride = row_stride_for(max_context_len, part, extra_row);

  pa::DecodeParams p{};
  p.q = q;
  p.k = cache->k;
  p.v = cache->v;
  p.out = out;
  p.tables = block_tables;
  p.lens = context_lens;
  if (need > 0) {
    const int64_t rows = (int64_t)num_seqs * num_q_heads * row_stride;
    char *w = static_cast<char *>(workspace);
    p.ws_m = reinterpret_cast<float *>(w);
    p.ws_l = reinterpret_cast<float *>(w + round16(rows * 4));
    p.ws_acc = reinterpret_cast<float *>(w + 2 * round16(rows * 4));
  }
  p.num_blocks = cache->num_blocks;
  p.Hkv = cache->num_kv_heads;
  p.bs = bs;
  p.Hq = num_q_heads;
  p.G = G;
  p.max_blocks = max_blocks_per_seq;
  p.B = num_seqs;
  p.max_ctx = max_context_len;
  p.max_parts = max_parts;
  p.row_stride = (int32_t)row_stride;
  p.part = part;
  p.scale_log2 = scale * 1.4426950408889634f;
  *pp = p;
  return PA_OK;
}

pa_status launch_decode_any(const pa::DecodeParams &p, const pa_cache_t *cache, cudaStream_t st) {
  if (tc_eligible(p, cache->dtype, cache->head_dim)) return launch_decode_tc(p, p.max_parts, st);
  if (cache->dtype == PA_DTYPE_F32) return launch_decode_dtype<float>(p, cache->head_dim, p.max_parts, st);
  return launch_decode_dtype<__nv_bfloat16>(p, cache->head_dim, p.max_parts, st);
}

}  // namespace

extern "C" {

PA_API pa_status pa_decode(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                           int32_t max_blocks_per_seq, const int32_t *context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
                           float scale, void *out, void *workspace, size_t workspace_bytes,
                           void *stream) {
  pa::DecodeParams p{};
  bool skip = false;
  const pa_status s = prepare_decode(q, cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                                     num_q_heads, max_context_len, scale, out, workspace,
                                     workspace_bytes, &p, &skip);
  if (s != PA_OK || skip) return s;
  return launch_decode_any(p, cache, (cudaStream_t)stream);
}

PA_API pa_status pa_append_decode(const void *k_new, const void *v_new, const int32_t *cow_src,
                                  const void *q, const pa_cache_t *cache,
                                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                                  const int32_t *context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t max_context_len, float scale,
                                  void *out, void *workspace, size_t workspace_bytes,
                                  void *stream) {
  pa::DecodeParams p{};
  bool skip = false;
  pa_status s = prepare_decode(q, cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                               num_q_heads, max_context_len, scale, out, workspace, workspace_bytes,
                               &p, &skip);
  if (s != PA_OK || skip) return s;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return PA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (tc_eligible(p, cache->dtype, cache->head_dim)) {
    p.k_new = k_new;
    p.v_new = v_new;
    p.cow_src = cow_src;
    return launch_decode_tc(p, p.max_parts, st);
  }
  // the CUDA-core decode does not append: a small kernel does it first
  const int row_vecs = cache->head_dim * elem_bytes(cache->dtype) / 16;
  const int64_t warps = (int64_t)num_seqs * cache->num_kv_heads;
  s = launch(pa::append_newest_kernel, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0, st,
             (const uint4 *)k_new, (const uint4 *)v_new, cow_src, block_tables, context_lens,
             max_blocks_per_seq, num_seqs, cache->num_kv_heads, cache->block_size, row_vecs,
             cache->num_blocks, max_context_len, (uint4 *)cache->k, (uint4 *)cache->v);
  if (s != PA_OK) return s;
  return launch_decode_any(p, cache, st);
}

PA_API pa_status pa_prefill(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                            int32_t max_blocks_per_seq, const int32_t *context_lens,
                            const int32_t *query_starts, int32_t num_seqs, int32_t num_q_heads,
                            int32_t total_query_tokens, int32_t max_query_len,
                            int32_t max_context_len, float scale, void *out, void *stream) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0 || max_blocks_per_seq < 0 ||
      total_query_tokens < 0 || max_query_len < 0)
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || total_query_tokens == 0) return PA_OK;
  if (!q || !out || !block_tables || !context_lens || !query_starts || !aligned16(q) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int32_t G = num_q_heads / cache->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (cache->dtype != PA_DTYPE_BF16 || cache->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * cache->block_size) return PA_ERR_INVALID_ARG;
  if (max_query_len > max_context_len) return PA_ERR_INVALID_ARG;
  if ((int64_t)cache->num_blocks * cache->num_kv_heads * cache->block_size >= (int64_t)INT32_MAX)
    return PA_ERR_INVALID_ARG;
  pa::DecodeParams p{};
  p.q = q;
  p.k = cache->k;
  p.v = cache->v;
  p.out = out;
  p.tables = block_tables;
  p.lens = context_lens;
  p.num_blocks = cache->num_blocks;
  p.Hkv = cache->num_kv_heads;
  p.bs = cache->block_size;
  p.Hq = num_q_heads;
  p.G = G;
  p.max_blocks = max_blocks_per_seq;
  p.B = num_seqs;
  p.max_ctx = max_context_len;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = (cudaStream_t)stream;
  switch (G) {
    case 1: return launch_prefill_g<1>(p, query_starts, total_query_tokens, max_query_len, st);
    case 2: return launch_prefill_g<2>(p, query_starts, total_query_tokens, max_query_len, st);
    case 4: return launch_prefill_g<4>(p, query_starts, total_query_tokens, max_query_len, st);
    default: return launch_prefill_g<8>(p, query_starts, total_query_tokens, max_query_len, st);
  }
}

PA_API pa_status pa_decode_shared(const void *k_new, const void *v_new, const int32_t *cow_src,
                                  const void *q, const pa_cache_t *cache,
                                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                                  const int32_t *context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t max_context_len, float scale,
                                  const pa_share_plan_t *plan, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream) {
  pa::DecodeParams p{};
  bool skip = false;
  const bool grouped = plan && plan->n_groups > 0;
  if (grouped && (!plan->members || !plan->shared_tokens || !plan->first_token ||
                  plan->max_members < 1 || plan->max_members > pa::ShLayout::kSlots))
    return PA_ERR_INVALID_ARG;
  pa_status s = prepare_decode(q, cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                               num_q_heads, max_context_len, scale, out, workspace, workspace_bytes,
                               &p, &skip, grouped);
  if (s != PA_OK || skip) return s;
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_INVALID_ARG;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return PA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (!tc_eligible(p, cache->dtype, cache->head_dim)) {
    // no cascade kernel on the CUDA-core path: every sequence computes all
    // of its partitions (the same result)
    if (k_new) {
      const int row_vecs = cache->head_dim * elem_bytes(cache->dtype) / 16;
      const int64_t warps = (int64_t)num_seqs * cache->num_kv_heads;
      s = launch(pa::append_newest_kernel, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0, st,
                 (const uint4 *)k_new, (const uint4 *)v_new, cow_src, block_tables, context_lens,
                 max_blocks_per_seq, num_seqs, cache->num_kv_heads, cache->block_size, row_vecs,
                 cache->num_blocks, max_context_len, (uint4 *)cache->k, (uint4 *)cache->v);
      if (s != PA_OK) return s;
    }
    return launch_decode_any(p, cache, st);
  }
  if (grouped) {
    s = launch_decode_shared(p, *plan, st);
    if (s != PA_OK) return s;
    p.first_tok = plan->first_token;
    p.late_wait = 1;
  }
  p.k_new = k_new;
  p.v_new = v_new;
  p.cow_src = k_new ? cow_src : nullptr;
  return launch_decode_tc(p, p.max_parts, st);
}

// ---------------------------------------------------------------------------
// pa_decode_static_workspace: pa_decode whose split-context scratch is this
// file-scope array instead of caller memory, for callers that cannot
// allocate device memory.  Host code must not use the array's name as a
// device address (it is a host-side stand-in); the device address comes from
// cudaGetSymbolAddress, looked up once per CUDA context with that context
// current and kept below.

}  // extern "C"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

// The array's device address differs between CUDA contexts (each context
// loads the module on its own), so the address looked up is kept per
// context, keyed by the context's unique id (cuCtxGetId: ids are never
// reused within a process, unlike context handles or device ordinals).  A
// context that is destroyed and re-created, e.g. after cudaDeviceReset,
// gets a new id and so a fresh lookup.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename Fn>
Fn driver_entry(const char *name) {
  void *f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(f);
}

constexpr int kStaticWsEntries = 64;
struct StaticWsEntry {
  unsigned long long ctx_id;
  void *ptr;
};
std::mutex g_static_ws_mutex;
StaticWsEntry g_static_ws[kStaticWsEntries] = {};
int g_static_ws_next = 0;  // the slot a new context takes (round-robin once all are used)

// Device address of the current context's copy of g_static_workspace, or
// nullptr (no context could be made current, or a lookup failed).
void *static_workspace_for_current_context() {
  static const CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return nullptr;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) {
    // no context bound to this thread yet: the runtime makes the current
    // device's primary context current (cudaSetDevice initialises it), then
    // ask again
    if (cudaSetDevice(dev) != cudaSuccess || get_current(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  for (const StaticWsEntry &e : g_static_ws)
    if (e.ptr && e.ctx_id == id) return e.ptr;
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess || !ptr) return nullptr;
  g_static_ws[g_static_ws_next] = StaticWsEntry{id, ptr};
  g_static_ws_next = (g_static_ws_next + 1) % kStaticWsEntries;
  return ptr;
}

}  // namespace

extern "C" {

PA_API pa_status pa_decode_static_workspace(const void *q, const pa_cache_t *cache,
                                            const int32_t *block_tables,
                                            int32_t max_blocks_per_seq,
                                            const int32_t *context_lens, int32_t num_seqs,
                                            int32_t num_q_heads, int32_t max_context_len,
                                            float scale, void *out, void *stream) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  // the range checks pa_decode makes, before the scratch size is computed
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0 || cache->head_dim <= 0)
    return PA_ERR_INVALID_ARG;
  const int32_t part = part_of(cache);
  if (num_seqs > 65535 || max_context_len > INT32_MAX - part) return PA_ERR_INVALID_ARG;
  const size_t need =
      num_seqs > 0 ? workspace_bytes_for(num_seqs, num_q_heads, max_context_len, cache->head_dim, part) : 0;
  if (need > (size_t)PA_STATIC_WORKSPACE_BYTES) return PA_ERR_TOO_SMALL;
  void *ws = nullptr;
  if (need > 0) {
    ws = static_workspace_for_current_context();
    if (!ws) return PA_ERR_CUDA;
  }
  return pa_decode(q, cache, block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                   max_context_len, scale, out, ws, need > 0 ? (size_t)PA_STATIC_WORKSPACE_BYTES : 0,
                   stream);
}

PA_API pa_status pa_read_wait_timeout(void *stream, uint32_t info[4]) {
  if (!info) return PA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
  uint32_t zero[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(info, pa::g_wait_timeout, sizeof zero) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyToSymbol(pa::g_wait_timeout, zero, sizeof zero) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

PA_API pa_status pa_read_device_error(void *stream, int32_t *bits) {
  if (!bits) return PA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_error, sizeof v) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyToSymbol(pa::g_error, &zero, sizeof zero) != cudaSuccess) return PA_ERR_CUDA;
  *bits = v;
  return PA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// One decode step from pinned host buffers: host work, one copy in, the
// decode, one copy out, ordered by the slot's events.

namespace {

inline size_t layout_take(size_t *at, size_t bytes) {
  const size_t off = *at;
  *at = round16(*at + bytes);
  return off;
}

}  // namespace

extern "C" {

PA_API pa_status pa_step_layout(int32_t n_seqs, int32_t num_q_heads, const pa_cache_t *cache,
                                int32_t max_blocks, int32_t share_max_members, pa_step_layout_t *layout) {
  if (!layout || !cache || n_seqs < 0 || num_q_heads <= 0 || max_blocks < 0 || share_max_members < 0 ||
      share_max_members > 4 || cache->num_kv_heads <= 0 || cache->head_dim <= 0)
    return PA_ERR_INVALID_ARG;
  if (cache->dtype != PA_DTYPE_F32 && cache->dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
  const size_t es = (size_t)elem_bytes(cache->dtype), n = (size_t)n_seqs, D = (size_t)cache->head_dim;
  const size_t groups = n / 2 > 0 ? n / 2 : 1;
  const size_t members = (size_t)(share_max_members > 0 ? share_max_members : 1);
  size_t at = 0;
  pa_step_layout_t L{};
  L.q = layout_take(&at, n * num_q_heads * D * es);
  L.k_new = layout_take(&at, n * cache->num_kv_heads * D * es);
  L.v_new = layout_take(&at, n * cache->num_kv_heads * D * es);
  L.tables = layout_take(&at, n * (size_t)max_blocks * 4);
  L.lens = layout_take(&at, n * 4);
  L.cow_src = layout_take(&at, n * 4);
  L.first_token = layout_take(&at, n * 4);
  L.members = layout_take(&at, groups * members * 4);
  L.shared_tokens = layout_take(&at, groups * 4);
  L.bytes = at;
  *layout = L;
  return PA_OK;
}

PA_API pa_status pa_step_slot_events(pa_step_slot_t *slot) {
  if (!slot) return PA_ERR_INVALID_ARG;
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
  for (int i = 0; i < 3; ++i) {
    const cudaError_t e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return cuda_failed(e);
    }
  }
  slot->ev_in = ev[0];
  slot->ev_kernel = ev[1];
  slot->ev_out = ev[2];
  return PA_OK;
}

PA_API pa_status pa_step_slot_release(pa_step_slot_t *slot) {
  if (!slot) return PA_ERR_INVALID_ARG;
  void **evs[3] = {&slot->ev_in, &slot->ev_kernel, &slot->ev_out};
  pa_status s = PA_OK;
  for (void **e : evs) {
    if (*e) {
      const cudaError_t r = cudaEventDestroy(static_cast<cudaEvent_t>(*e));
      if (r != cudaSuccess) s = cuda_failed(r);
      *e = nullptr;
    }
  }
  return s;
}

PA_API pa_status pa_step_slot_wait(const pa_step_slot_t *slot) {
  if (!slot || !slot->ev_in || !slot->ev_out) return PA_ERR_INVALID_ARG;
  cudaError_t e = cudaEventSynchronize(static_cast<cudaEvent_t>(slot->ev_in));
  if (e == cudaSuccess) e = cudaEventSynchronize(static_cast<cudaEvent_t>(slot->ev_out));
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

PA_API pa_status pa_decode_step(pa_allocator *a, const int32_t *seqs_host, int32_t n_seqs,
                                int32_t max_blocks, int32_t share_max_members,
                                const pa_cache_t *cache, int32_t num_q_heads, float scale,
                                const pa_step_slot_t *slot, void *stream, void *h2d_stream,
                                void *d2h_stream,
                                int32_t *n_copies, int32_t *n_groups, int32_t *max_len) {
  if (!a || !slot || !n_copies || !n_groups || !max_len || !slot->host || !slot->dev || !slot->out_host ||
      !slot->out_dev || !slot->ev_in || !slot->ev_kernel || !slot->ev_out)
    return PA_ERR_INVALID_ARG;
  pa_step_layout_t L{};
  pa_status s = pa_step_layout(n_seqs, num_q_heads, cache, max_blocks, share_max_members, &L);
  if (s != PA_OK) return s;
  s = check_cache(cache);
  if (s != PA_OK) return s;
  if (!aligned16(slot->host) || !aligned16(slot->dev)) return PA_ERR_INVALID_ARG;
  // the decode's own checks, before the allocator moves (a step too long
  // for the table width is refused by the preparation itself)
  if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int64_t ctx_cap = (int64_t)max_blocks * cache->block_size;
  const int32_t part = part_of(cache);
  if (ctx_cap > INT32_MAX - part) return PA_ERR_INVALID_ARG;
  const size_t need_ws =
      n_seqs > 0 ? workspace_bytes_for(n_seqs, num_q_heads, (int32_t)ctx_cap, cache->head_dim, part,
                                       share_max_members > 0)
                 : 0;
  if (need_ws > 0 && (!slot->workspace || slot->workspace_bytes < need_ws)) return PA_ERR_TOO_SMALL;
  char *h = static_cast<char *>(slot->host);
  char *d = static_cast<char *>(slot->dev);
  auto hi = [&](size_t off) { return reinterpret_cast<int32_t *>(h + off); };
  auto di = [&](size_t off) { return reinterpret_cast<int32_t *>(d + off); };
  s = pa_decode_step_prepare(a, seqs_host, n_seqs, max_blocks, share_max_members, hi(L.tables), hi(L.lens),
                             hi(L.cow_src), hi(L.members), hi(L.shared_tokens), hi(L.first_token), n_groups,
                             n_copies, max_len);
  if (s != PA_OK || n_seqs == 0) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t hst = static_cast<cudaStream_t>(h2d_stream);
  cudaStream_t dst = static_cast<cudaStream_t>(d2h_stream);
  cudaEvent_t ev_in = static_cast<cudaEvent_t>(slot->ev_in);
  cudaEvent_t ev_kernel = static_cast<cudaEvent_t>(slot->ev_kernel);
  cudaEvent_t ev_out = static_cast<cudaEvent_t>(slot->ev_out);
  cudaError_t e;
  // inputs: after the slot's previous decode has read its device copy
  if ((e = cudaStreamWaitEvent(hst, ev_kernel, 0)) != cudaSuccess) return cuda_failed(e);
  if ((e = cudaMemcpyAsync(d, h, L.bytes, cudaMemcpyHostToDevice, hst)) != cudaSuccess) return cuda_failed(e);
  if ((e = cudaEventRecord(ev_in, hst)) != cudaSuccess) return cuda_failed(e);
  // the decode: after the inputs, and after the previous output left out_dev
  if ((e = cudaStreamWaitEvent(st, ev_in, 0)) != cudaSuccess) return cuda_failed(e);
  if ((e = cudaStreamWaitEvent(st, ev_out, 0)) != cudaSuccess) return cuda_failed(e);
  pa_share_plan_t plan{di(L.members), di(L.shared_tokens), di(L.first_token), *n_groups,
                       share_max_members > 0 ? share_max_members : 1};
  s = pa_decode_shared(d + L.k_new, d + L.v_new, *n_copies > 0 ? di(L.cow_src) : nullptr, d + L.q, cache,
                       di(L.tables), max_blocks, di(L.lens), n_seqs, num_q_heads, *max_len, scale,
                       *n_groups > 0 ? &plan : nullptr, slot->out_dev, slot->workspace, slot->workspace_bytes,
                       stream);
  if (s != PA_OK) return s;
  if ((e = cudaEventRecord(ev_kernel, st)) != cudaSuccess) return cuda_failed(e);
  // the output, back to the host
  if ((e = cudaStreamWaitEvent(dst, ev_kernel, 0)) != cudaSuccess) return cuda_failed(e);
  const size_t out_bytes = (size_t)n_seqs * num_q_heads * cache->head_dim * elem_bytes(cache->dtype);
  if ((e = cudaMemcpyAsync(slot->out_host, slot->out_dev, out_bytes, cudaMemcpyDeviceToHost, dst)) != cudaSuccess)
    return cuda_failed(e);
  if ((e = cudaEventRecord(ev_out, dst)) != cudaSuccess) return cuda_failed(e);
  return PA_OK;
}

}  // extern "C"

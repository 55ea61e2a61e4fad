// Host-side block allocator of the paged KV cache.
//
// "PagedAttention Internals" (wondering.app), "Fixed-Size KV Blocks": a
// sequence starts with no reservation, tokens fill its current block and a
// block is taken only when that one is full, so waste is confined to the last
// block; "Sharing And Dynamic Growth": blocks are obtained as needed and
// released when a request finishes.  "pagedattention" glossary entry
// (chipfoundryservices.com), comparison table and paragraph "It is the core of
// vLLM ...": sequences sharing a prompt prefix or the samples of a beam
// search point at the same physical blocks and fork copy-on-write only when
// they diverge.
//
// Design: a flat reference-count array over the pool, a LIFO free stack
// (fresh blocks dealt in a caller-given order, released blocks reused first
// while they are still warm in L2), and per-sequence std::vector tables.
// Appends are all-or-nothing: a dry run counts the blocks a batch needs
// (fresh blocks plus copy-on-write moves) before anything changes.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int32_t len = 0;
  bool live = false;
};

}  // namespace

struct pa_allocator {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // top = back
  std::vector<int32_t> ref;
  std::vector<Seq> seqs;
  // scratch of the dry run: reference counts a batch will have given up
  std::vector<int32_t> taken;
  std::vector<int32_t> touched;

  Seq *find(int32_t id) {
    if (id < 0 || id >= (int32_t)seqs.size() || !seqs[id].live) return nullptr;
    return &seqs[id];
  }

  static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

  // Blocks an append of n tokens to s will take, given the reference counts
  // earlier members of the same batch have already given up.
  int64_t blocks_needed(const Seq &s, int32_t n) {
    if (n <= 0) return 0;
    int64_t pos = s.len;
    int64_t need = ceil_div(pos + n, block_size) - ceil_div(pos, block_size);
    if (pos % block_size) {
      int32_t last = s.table.back();
      if (ref[last] - taken[last] > 1) {
        if (taken[last] == 0) touched.push_back(last);
        ++taken[last];
        ++need;
      }
    }
    return need;
  }

  void clear_taken() {
    for (int32_t b : touched) taken[b] = 0;
    touched.clear();
  }

  int32_t pop_free() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    return b;
  }

  // Executes an append whose blocks were already counted.
  void do_append(Seq &s, int32_t n, int64_t *slots, int32_t *cow_pair, int32_t *n_cow) {
    const int32_t bs = block_size;
    for (int32_t i = 0; i < n; ++i) {
      int32_t pos = s.len;
      if (pos % bs == 0) {
        int32_t b = pop_free();
        ref[b] = 1;
        s.table.push_back(b);
      } else {
        int32_t last = s.table.back();
        if (ref[last] > 1) {
          int32_t fresh = pop_free();
          ref[fresh] = 1;
          --ref[last];
          s.table.back() = fresh;
          cow_pair[0] = last;
          cow_pair[1] = fresh;
          ++*n_cow;
        }
      }
      slots[i] = (int64_t)s.table[pos / bs] * bs + pos % bs;
      s.len = pos + 1;
    }
  }
};

extern "C" {

PA_API pa_status pa_alloc_create(int32_t num_blocks, int32_t block_size,
                                 const int32_t *free_order_host, pa_allocator **out) {
  if (!out || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  pa_allocator *a = new (std::nothrow) pa_allocator();
  if (!a) return PA_ERR_INVALID_ARG;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ref.assign(num_blocks, 0);
  a->taken.assign(num_blocks, 0);
  a->free_stack.resize(num_blocks);
  if (free_order_host) {
    std::vector<uint8_t> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      int32_t b = free_order_host[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return PA_ERR_INVALID_ARG;
      }
      seen[b] = 1;
      a->free_stack[num_blocks - 1 - i] = b;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->free_stack[num_blocks - 1 - i] = i;
  }
  *out = a;
  return PA_OK;
}

PA_API void pa_alloc_destroy(pa_allocator *a) { delete a; }

PA_API pa_status pa_seq_new(pa_allocator *a, int32_t *seq) {
  if (!a || !seq) return PA_ERR_INVALID_ARG;
  if (a->seqs.size() >= (size_t)INT32_MAX) return PA_ERR_INVALID_ARG;
  a->seqs.emplace_back();
  a->seqs.back().live = true;
  *seq = (int32_t)a->seqs.size() - 1;
  return PA_OK;
}

PA_API pa_status pa_seq_fork(pa_allocator *a, int32_t parent, int32_t *child) {
  if (!a || !child) return PA_ERR_INVALID_ARG;
  if (!a->find(parent)) return PA_ERR_NOT_FOUND;
  int32_t id;
  pa_status st = pa_seq_new(a, &id);
  if (st != PA_OK) return st;
  Seq &p = a->seqs[parent];  // re-fetch: emplace_back may have moved it
  Seq &c = a->seqs[id];
  c.table = p.table;
  c.len = p.len;
  for (int32_t b : c.table) ++a->ref[b];
  *child = id;
  return PA_OK;
}

PA_API pa_status pa_seq_free(pa_allocator *a, int32_t seq) {
  if (!a) return PA_ERR_INVALID_ARG;
  Seq *s = a->find(seq);
  if (!s) return PA_ERR_NOT_FOUND;
  for (int32_t b : s->table) {
    if (--a->ref[b] == 0) a->free_stack.push_back(b);
  }
  s->table.clear();
  s->table.shrink_to_fit();
  s->len = 0;
  s->live = false;
  return PA_OK;
}

PA_API pa_status pa_seq_append(pa_allocator *a, int32_t seq, int32_t n, int64_t *out_slots_host,
                               int32_t *out_cow_pair_host, int32_t *n_cow) {
  return pa_batch_append(a, &seq, &n, 1, out_slots_host, out_cow_pair_host, n_cow);
}

PA_API pa_status pa_batch_append(pa_allocator *a, const int32_t *seqs, const int32_t *n_tokens,
                                 int32_t n_seqs, int64_t *out_slots_host,
                                 int32_t *out_cow_pairs_host, int32_t *n_cow) {
  if (!a || n_seqs < 0 || !n_cow || (n_seqs > 0 && (!seqs || !n_tokens))) return PA_ERR_INVALID_ARG;
  *n_cow = 0;
  int64_t total = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    if (n_tokens[i] < 0) return PA_ERR_INVALID_ARG;
    if (!a->find(seqs[i])) return PA_ERR_NOT_FOUND;
    if ((int64_t)a->seqs[seqs[i]].len + n_tokens[i] > INT32_MAX) return PA_ERR_INVALID_ARG;
    total += n_tokens[i];
  }
  if (total > 0 && !out_slots_host) return PA_ERR_INVALID_ARG;
  if (n_seqs > 0 && !out_cow_pairs_host) return PA_ERR_INVALID_ARG;
  // a sequence may appear at most once per batch
  if (n_seqs > 1) {
    std::vector<int32_t> ids(seqs, seqs + n_seqs);
    std::sort(ids.begin(), ids.end());
    if (std::adjacent_find(ids.begin(), ids.end()) != ids.end()) return PA_ERR_INVALID_ARG;
  }
  int64_t need = 0;
  for (int32_t i = 0; i < n_seqs; ++i) need += a->blocks_needed(a->seqs[seqs[i]], n_tokens[i]);
  a->clear_taken();
  if (need > (int64_t)a->free_stack.size()) return PA_ERR_OUT_OF_BLOCKS;
  int64_t off = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    int32_t made = 0;
    a->do_append(a->seqs[seqs[i]], n_tokens[i], out_slots_host + off,
                 out_cow_pairs_host + 2 * (*n_cow), &made);
    *n_cow += made;
    off += n_tokens[i];
  }
  return PA_OK;
}

PA_API pa_status pa_seq_len(pa_allocator *a, int32_t seq, int32_t *len, int32_t *num_blocks) {
  if (!a) return PA_ERR_INVALID_ARG;
  Seq *s = a->find(seq);
  if (!s) return PA_ERR_NOT_FOUND;
  if (len) *len = s->len;
  if (num_blocks) *num_blocks = (int32_t)s->table.size();
  return PA_OK;
}

PA_API pa_status pa_seq_block_table(pa_allocator *a, int32_t seq, int32_t *out_host, int32_t cap,
                                    int32_t *count) {
  if (!a || !count || cap < 0 || (cap > 0 && !out_host)) return PA_ERR_INVALID_ARG;
  Seq *s = a->find(seq);
  if (!s) return PA_ERR_NOT_FOUND;
  *count = (int32_t)s->table.size();
  if (*count > cap) return PA_ERR_TOO_SMALL;
  if (*count) std::memcpy(out_host, s->table.data(), sizeof(int32_t) * (size_t)*count);
  return PA_OK;
}

PA_API pa_status pa_seqs_max_len(pa_allocator *a, const int32_t *seqs, int32_t n_seqs,
                                 int32_t *max_len, int32_t *max_blocks) {
  if (!a || n_seqs < 0 || (n_seqs > 0 && !seqs) || !max_len || !max_blocks) return PA_ERR_INVALID_ARG;
  int32_t ml = 0, mb = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq *s = a->find(seqs[i]);
    if (!s) return PA_ERR_NOT_FOUND;
    if (s->len > ml) ml = s->len;
    if ((int32_t)s->table.size() > mb) mb = (int32_t)s->table.size();
  }
  *max_len = ml;
  *max_blocks = mb;
  return PA_OK;
}

PA_API pa_status pa_build_block_tables(pa_allocator *a, const int32_t *seqs, int32_t n_seqs,
                                       int32_t max_blocks, int32_t pad, int32_t *tables_host,
                                       int32_t *lens_host) {
  if (!a || n_seqs < 0 || max_blocks < 0) return PA_ERR_INVALID_ARG;
  if (n_seqs > 0 && (!seqs || !lens_host || (max_blocks > 0 && !tables_host)))
    return PA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n_seqs; ++i) {
    Seq *s = a->find(seqs[i]);
    if (!s) return PA_ERR_NOT_FOUND;
    if ((int32_t)s->table.size() > max_blocks) return PA_ERR_TOO_SMALL;
  }
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq &s = a->seqs[seqs[i]];
    int32_t *row = tables_host + (int64_t)i * max_blocks;
    int32_t nb = (int32_t)s.table.size();
    if (nb) std::memcpy(row, s.table.data(), sizeof(int32_t) * (size_t)nb);
    for (int32_t j = nb; j < max_blocks; ++j) row[j] = pad;
    lens_host[i] = s.len;
  }
  return PA_OK;
}

PA_API pa_status pa_alloc_stats(pa_allocator *a, int64_t *used_slots, int64_t *allocated_slots,
                                int32_t *free_blocks, int32_t *used_blocks) {
  if (!a) return PA_ERR_INVALID_ARG;
  int32_t used_b = a->num_blocks - (int32_t)a->free_stack.size();
  if (used_slots) {
    // every physical slot once: a shared block has the same fill for every
    // sharer (a write into a shared partial block moves the writer first)
    std::vector<int32_t> fill(a->num_blocks, -1);
    int64_t used = 0;
    const int32_t bs = a->block_size;
    for (const Seq &s : a->seqs) {
      if (!s.live) continue;
      for (size_t j = 0; j < s.table.size(); ++j) {
        int32_t b = s.table[j];
        if (fill[b] < 0) {
          int64_t f = (int64_t)s.len - (int64_t)j * bs;
          fill[b] = (int32_t)(f < bs ? f : bs);
          used += fill[b];
        }
      }
    }
    *used_slots = used;
  }
  if (allocated_slots) *allocated_slots = (int64_t)used_b * a->block_size;
  if (free_blocks) *free_blocks = (int32_t)a->free_stack.size();
  if (used_blocks) *used_blocks = used_b;
  return PA_OK;
}

PA_API pa_status pa_block_refcount(pa_allocator *a, int32_t block, int32_t *refcount) {
  if (!a || !refcount || block < 0 || block >= a->num_blocks) return PA_ERR_INVALID_ARG;
  *refcount = a->ref[block];
  return PA_OK;
}

PA_API pa_status pa_share_plan(const int32_t *tables_host, int32_t max_blocks,
                               const int32_t *lens_host, int32_t n_seqs, int32_t block_size,
                               int32_t max_members, int32_t *members_host, int32_t *shared_host,
                               int32_t *first_token_host, int32_t *n_groups) {
  if (n_seqs < 0 || max_blocks < 0 || !n_groups || max_members < 2 || max_members > 4 ||
      (block_size != 8 && block_size != 16 && block_size != 32))
    return PA_ERR_INVALID_ARG;
  if (n_seqs > 0 && (!tables_host || !lens_host || !members_host || !shared_host || !first_token_host))
    return PA_ERR_INVALID_ARG;
  *n_groups = 0;
  for (int32_t b = 0; b < n_seqs; ++b) first_token_host[b] = 0;
  auto row = [&](int32_t b) { return tables_host + (size_t)b * max_blocks; };
  auto nblocks = [&](int32_t b) { return (int32_t)(((int64_t)lens_host[b] + block_size - 1) / block_size); };
  // sequences with a block before their last one: only such blocks can be
  // shared (a sequence's last block is the one it writes)
  std::vector<int32_t> cand;
  for (int32_t b = 0; b < n_seqs; ++b) {
    const int32_t nb = nblocks(b);
    if (lens_host[b] > 0 && nb >= 2 && nb <= max_blocks) cand.push_back(b);
  }
  // buckets: the same first physical block (sharers point at the same blocks
  // from the start), sequence order inside a bucket; buckets in the order of
  // their first (lowest) sequence index
  std::stable_sort(cand.begin(), cand.end(), [&](int32_t x, int32_t y) { return row(x)[0] < row(y)[0]; });
  std::vector<std::pair<size_t, size_t>> runs;
  for (size_t i = 0; i < cand.size();) {
    size_t e = i + 1;
    while (e < cand.size() && row(cand[e])[0] == row(cand[i])[0]) ++e;
    runs.emplace_back(i, e);
    i = e;
  }
  std::sort(runs.begin(), runs.end(), [&](const std::pair<size_t, size_t> &x, const std::pair<size_t, size_t> &y) {
    return cand[x.first] < cand[y.first];
  });
  for (const auto &run : runs) {
    for (size_t g0 = run.first; g0 + 1 < run.second; g0 += (size_t)max_members) {
      const size_t g1 = std::min(run.second, g0 + (size_t)max_members);
      if (g1 - g0 < 2) break;  // a lone leftover shares with nobody
      // leading blocks on which every member agrees, each before every
      // member's last block
      int32_t lim = INT32_MAX;
      for (size_t k = g0; k < g1; ++k) lim = std::min(lim, nblocks(cand[k]) - 1);
      int32_t nshared = 0;
      const int32_t *r0 = row(cand[g0]);
      while (nshared < lim) {
        bool same = true;
        for (size_t k = g0 + 1; k < g1 && same; ++k) same = row(cand[k])[nshared] == r0[nshared];
        if (!same) break;
        ++nshared;
      }
      const int32_t tokens = nshared * block_size;
      if (tokens < PA_SHARE_MIN_TOKENS) continue;
      int32_t *mem = members_host + (size_t)(*n_groups) * max_members;
      for (int32_t k = 0; k < max_members; ++k) mem[k] = g0 + k < g1 ? cand[g0 + k] : -1;
      shared_host[*n_groups] = tokens;
      for (size_t k = g0; k < g1; ++k) first_token_host[cand[k]] = tokens;
      ++*n_groups;
    }
  }
  return PA_OK;
}

PA_API pa_status pa_decode_step_prepare(pa_allocator *a, const int32_t *seqs, int32_t n_seqs,
                                        int32_t max_blocks, int32_t share_max_members,
                                        int32_t *tables_host, int32_t *lens_host,
                                        int32_t *cow_src_host, int32_t *members_host,
                                        int32_t *shared_host, int32_t *first_token_host,
                                        int32_t *n_groups, int32_t *n_copies, int32_t *max_len) {
  if (!a || n_seqs < 0 || max_blocks < 0 || !n_groups || !n_copies || !max_len) return PA_ERR_INVALID_ARG;
  if (n_seqs > 0 && (!seqs || !tables_host || !lens_host || !cow_src_host || !first_token_host))
    return PA_ERR_INVALID_ARG;
  if (share_max_members != 0 &&
      (share_max_members < 2 || share_max_members > 4 || (n_seqs > 1 && (!members_host || !shared_host))))
    return PA_ERR_INVALID_ARG;
  *n_groups = 0;
  *n_copies = 0;
  *max_len = 0;
  const int32_t bs = a->block_size;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq *s = a->find(seqs[i]);
    if (!s) return PA_ERR_NOT_FOUND;
    if (s->len == INT32_MAX) return PA_ERR_INVALID_ARG;
    if (pa_allocator::ceil_div((int64_t)s->len + 1, bs) > max_blocks) return PA_ERR_TOO_SMALL;
  }
  if (n_seqs > 1) {  // a sequence may appear once
    std::vector<int32_t> ids(seqs, seqs + n_seqs);
    std::sort(ids.begin(), ids.end());
    if (std::adjacent_find(ids.begin(), ids.end()) != ids.end()) return PA_ERR_INVALID_ARG;
  }
  // one token per sequence, all or nothing
  int64_t need = 0;
  for (int32_t i = 0; i < n_seqs; ++i) need += a->blocks_needed(a->seqs[seqs[i]], 1);
  a->clear_taken();
  if (need > (int64_t)a->free_stack.size()) return PA_ERR_OUT_OF_BLOCKS;
  for (int32_t i = 0; i < n_seqs; ++i) {
    int64_t slot;
    int32_t pair[2] = {-1, -1};
    int32_t made = 0;
    a->do_append(a->seqs[seqs[i]], 1, &slot, pair, &made);
    cow_src_host[i] = made ? pair[0] : -1;  // the copy lands in the sequence's (new) last block
    *n_copies += made;
  }
  // the tables (entries past a sequence's blocks are not written: no kernel
  // reads them) and lengths
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq &s = a->seqs[seqs[i]];
    const size_t nb = s.table.size();
    if (nb) std::memcpy(tables_host + (int64_t)i * max_blocks, s.table.data(), sizeof(int32_t) * nb);
    lens_host[i] = s.len;
    *max_len = std::max(*max_len, s.len);
  }
  if (share_max_members == 0) {
    for (int32_t i = 0; i < n_seqs; ++i) first_token_host[i] = 0;
    return PA_OK;
  }
  return pa_share_plan(tables_host, max_blocks, lens_host, n_seqs, bs, share_max_members, members_host,
                       shared_host, first_token_host, n_groups);
}

PA_API pa_status pa_cow_sources(const int32_t *pairs_host, int32_t n_pairs,
                                const int32_t *tables_host, int32_t max_blocks,
                                const int32_t *lens_host, int32_t n_seqs, int32_t block_size,
                                int32_t *cow_src_host) {
  if (n_pairs < 0 || n_seqs < 0 || max_blocks < 0 || block_size <= 0 || (n_pairs > 0 && !pairs_host) ||
      (n_seqs > 0 && (!tables_host || !lens_host || !cow_src_host)))
    return PA_ERR_INVALID_ARG;
  std::unordered_map<int32_t, int32_t> src_of;  // destination -> source
  src_of.reserve((size_t)n_pairs * 2);
  for (int32_t i = 0; i < n_pairs; ++i)
    if (!src_of.emplace(pairs_host[2 * i + 1], pairs_host[2 * i]).second) return PA_ERR_INVALID_ARG;
  int32_t matched = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    cow_src_host[i] = -1;
    const int32_t len = lens_host[i];
    if (len <= 0) continue;  // no last block
    const int64_t col = (int64_t)(len - 1) / block_size;  // the table entry of the newest token
    if (col >= max_blocks) return PA_ERR_INVALID_ARG;
    auto it = src_of.find(tables_host[(int64_t)i * max_blocks + col]);
    if (it == src_of.end()) continue;
    cow_src_host[i] = it->second;
    src_of.erase(it);  // one writer per destination
    ++matched;
  }
  return matched == n_pairs ? PA_OK : PA_ERR_INVALID_ARG;
}

PA_API pa_status pa_alloc_fragmentation(pa_allocator *a, double *fragmentation) {
  if (!a || !fragmentation) return PA_ERR_INVALID_ARG;
  int64_t used = 0, allocated = 0;
  const pa_status s = pa_alloc_stats(a, &used, &allocated, nullptr, nullptr);
  if (s != PA_OK) return s;
  // waste over what is held: (allocated - used) / allocated
  *fragmentation = allocated > 0 ? (double)(allocated - used) / (double)allocated : 0.0;
  return PA_OK;
}

}  // extern "C"

// Host page bookkeeping for the paged K/V cache (declared in include/gqa_pager.h).
//
// The tiny-llm "优化" page preallocates the cache once and pages it through a block
// table; continuous batching is its scheduler-side next step.  Here: a free list of pool
// page ids (a stack: the last page freed is the first reused), and per sequence slot its
// length and its pages in token order (a row of a [max_seqs, max_blocks] table, -1 past
// its pages).  Every mutating call checks everything first and then applies, so an error
// changes nothing.
#include <cstdint>
#include <new>
#include <vector>

#include "gqa_pager.h"
#include "internal.cuh"

struct gqa_pager {
  int num_pages = 0, page_size = 0, max_seqs = 0, max_blocks = 0;
  std::vector<int32_t> free_list;  // top = back()
  std::vector<int32_t> table;      // [max_seqs * max_blocks]
  std::vector<int32_t> lens;       // [max_seqs]
  std::vector<uint8_t> mark;       // [max_seqs] scratch for duplicate checks
};

namespace {

int64_t blocks_for(int64_t len, int ps) { return (len + ps - 1) / ps; }

bool bad_slot(const gqa_pager* g, int seq) { return seq < 0 || seq >= g->max_seqs; }

// Pages slot `seq` needs to hold `new_len` tokens, or -1 beyond max_blocks.
int64_t needed_pages(const gqa_pager* g, int seq, int64_t new_len) {
  const int64_t nb = blocks_for(new_len, g->page_size);
  if (nb > g->max_blocks) return -1;
  return nb - blocks_for(g->lens[seq], g->page_size);
}

void grow(gqa_pager* g, int seq, int64_t new_len) {
  int32_t* row = g->table.data() + static_cast<int64_t>(seq) * g->max_blocks;
  for (int64_t b = blocks_for(g->lens[seq], g->page_size); b < blocks_for(new_len, g->page_size); ++b) {
    row[b] = g->free_list.back();
    g->free_list.pop_back();
  }
  g->lens[seq] = static_cast<int32_t>(new_len);
}

}  // namespace

extern "C" {

gqa_status gqa_pager_create(int num_pages, int page_size, int max_seqs, int max_blocks_per_seq,
                            gqa_pager** out) {
  if (!out) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_create: out is NULL");
  *out = nullptr;
  if (num_pages < 0 || page_size <= 0 || max_seqs < 0 || max_blocks_per_seq <= 0)
    return gqa::set_error(GQA_ERR_INVALID_ARG,
                          "gqa_pager_create: need num_pages >= 0, page_size > 0, max_seqs >= 0, "
                          "max_blocks_per_seq > 0 (got %d, %d, %d, %d)",
                          num_pages, page_size, max_seqs, max_blocks_per_seq);
  if (static_cast<int64_t>(max_blocks_per_seq) * page_size > INT32_MAX)
    return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_create: max_blocks_per_seq * page_size overflows int32");
  gqa_pager* g = new (std::nothrow) gqa_pager;
  if (!g) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_create: out of host memory");
  try {
    g->num_pages = num_pages;
    g->page_size = page_size;
    g->max_seqs = max_seqs;
    g->max_blocks = max_blocks_per_seq;
    g->free_list.resize(num_pages);
    for (int i = 0; i < num_pages; ++i) g->free_list[i] = num_pages - 1 - i;  // page 0 on top
    g->table.assign(static_cast<size_t>(max_seqs) * max_blocks_per_seq, -1);
    g->lens.assign(max_seqs, 0);
    g->mark.assign(max_seqs, 0);
  } catch (...) {
    delete g;
    return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_create: out of host memory");
  }
  *out = g;
  return GQA_OK;
}

void gqa_pager_destroy(gqa_pager* pager) { delete pager; }

gqa_status gqa_pager_extend(gqa_pager* g, int seq, int n_tokens) {
  if (!g) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_extend: pager is NULL");
  if (bad_slot(g, seq) || n_tokens < 0)
    return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_extend: slot %d / count %d out of range", seq, n_tokens);
  const int64_t new_len = static_cast<int64_t>(g->lens[seq]) + n_tokens;
  const int64_t need = needed_pages(g, seq, new_len);
  if (need < 0)
    return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_extend: %lld tokens exceed max_blocks_per_seq * page_size",
                          static_cast<long long>(new_len));
  if (need > static_cast<int64_t>(g->free_list.size()))
    return gqa::set_error(GQA_ERR_OUT_OF_PAGES, "gqa_pager_extend: %lld pages needed, %zu free",
                          static_cast<long long>(need), g->free_list.size());
  grow(g, seq, new_len);
  return GQA_OK;
}

gqa_status gqa_pager_step(gqa_pager* g, const int32_t* seqs, int n, int32_t* positions, int32_t* seq_lens) {
  if (!g) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_step: pager is NULL");
  if (n < 0 || (n > 0 && !seqs)) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_step: bad batch");
  int64_t need = 0;
  gqa_status st = GQA_OK;
  int i = 0;
  for (; i < n; ++i) {
    const int s = seqs[i];
    if (bad_slot(g, s)) {
      st = gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_step: slot %d out of range", s);
      break;
    }
    if (g->mark[s]) {
      st = gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_step: slot %d listed twice", s);
      break;
    }
    g->mark[s] = 1;
    const int64_t d = needed_pages(g, s, static_cast<int64_t>(g->lens[s]) + 1);
    if (d < 0) {
      st = gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_step: slot %d is full (max_blocks_per_seq)", s);
      break;
    }
    need += d;
  }
  for (int j = 0; j < i + (st == GQA_OK ? 0 : 1) && j < n; ++j)
    if (!bad_slot(g, seqs[j])) g->mark[seqs[j]] = 0;
  if (st != GQA_OK) return st;
  if (need > static_cast<int64_t>(g->free_list.size()))
    return gqa::set_error(GQA_ERR_OUT_OF_PAGES, "gqa_pager_step: %lld pages needed, %zu free",
                          static_cast<long long>(need), g->free_list.size());
  for (int j = 0; j < n; ++j) {
    const int s = seqs[j];
    if (positions) positions[j] = g->lens[s];
    grow(g, s, static_cast<int64_t>(g->lens[s]) + 1);
    if (seq_lens) seq_lens[j] = g->lens[s];
  }
  return GQA_OK;
}

gqa_status gqa_pager_truncate(gqa_pager* g, int seq, int new_len) {
  if (!g) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_truncate: pager is NULL");
  if (bad_slot(g, seq) || new_len < 0 || new_len > g->lens[seq])
    return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_truncate: slot %d / length %d out of range", seq, new_len);
  int32_t* row = g->table.data() + static_cast<int64_t>(seq) * g->max_blocks;
  // Freed in reverse block order, so the slot's first page ends on top of the stack.
  for (int64_t b = blocks_for(g->lens[seq], g->page_size) - 1; b >= blocks_for(new_len, g->page_size); --b) {
    g->free_list.push_back(row[b]);
    row[b] = -1;
  }
  g->lens[seq] = new_len;
  return GQA_OK;
}

gqa_status gqa_pager_gather(const gqa_pager* g, const int32_t* seqs, int n, int32_t* block_table,
                            int32_t* seq_lens) {
  if (!g) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_gather: pager is NULL");
  if (n < 0 || (n > 0 && !seqs)) return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_gather: bad batch");
  for (int i = 0; i < n; ++i)
    if (bad_slot(g, seqs[i]))
      return gqa::set_error(GQA_ERR_INVALID_ARG, "gqa_pager_gather: slot %d out of range", seqs[i]);
  for (int i = 0; i < n; ++i) {
    const int s = seqs[i];
    if (block_table) {
      const int32_t* row = g->table.data() + static_cast<int64_t>(s) * g->max_blocks;
      int32_t* dst = block_table + static_cast<int64_t>(i) * g->max_blocks;
      for (int b = 0; b < g->max_blocks; ++b) dst[b] = row[b];
    }
    if (seq_lens) seq_lens[i] = g->lens[s];
  }
  return GQA_OK;
}

int gqa_pager_free_pages(const gqa_pager* g) { return g ? static_cast<int>(g->free_list.size()) : -1; }

int gqa_pager_seq_len(const gqa_pager* g, int seq) { return (!g || bad_slot(g, seq)) ? -1 : g->lens[seq]; }

}  // extern "C"

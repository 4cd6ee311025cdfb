// Paged KV-cache bookkeeping (host): a pool of fixed-size pages of token slots and,
// per sequence, the block table of the pages its tokens occupy in order.
//
// "TurboQuant + RotorQuant", "Post-Prefill Quantization": the prefill cache is
// quantized in bulk at the first decode step and every later step quantizes one new
// key and value for storage. With many sequences of different lengths those
// packed rows live in pages: logical token t of a sequence sits in slot
// page_tokens * table[t / page_tokens] + t % page_tokens of the pool, so the bulk
// pass writes whole pages and each decode step writes one slot. This file keeps
// only the bookkeeping; the packed rows themselves are device memory of the caller,
// indexed by these slot numbers.

#include <cstdint>
#include <memory>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "kvrq.h"
#include "kvrq_internal.h"

struct kvrq_pages {
  int64_t n_pages = 0;
  int page_tokens = 0;
  std::vector<int32_t> free_list;  // pages not in any block table (popped from the back)
  struct Seq {
    std::vector<int32_t> table;
    int64_t tokens = 0;
  };
  std::unordered_map<int64_t, Seq> seqs;
  int64_t next_id = 0;
  std::mutex mu;
};

using namespace kvrq;

extern "C" {

kvrq_status kvrq_pages_create(int64_t n_pages, int page_tokens, kvrq_pages** out) {
  if (!out) return set_error(KVRQ_EINVAL, "kvrq_pages_create: out is NULL");
  *out = nullptr;
  if (n_pages < 1 || n_pages > INT32_MAX || page_tokens < 1)
    return set_error(KVRQ_EINVAL, "kvrq_pages_create: n_pages in 1..2^31-1 and page_tokens >= 1");
  return guarded("kvrq_pages_create", [&] {
    alloc_check();
    std::unique_ptr<kvrq_pages> p(new kvrq_pages());
    p->n_pages = n_pages;
    p->page_tokens = page_tokens;
    // the free list never holds more than n_pages pages: later pushes never reallocate
    p->free_list.reserve((size_t)n_pages);
    for (int64_t i = n_pages - 1; i >= 0; --i) p->free_list.push_back((int32_t)i);  // page 0 is handed out first
    *out = p.release();
    return KVRQ_OK;
  });
}

void kvrq_pages_destroy(kvrq_pages* p) { delete p; }

kvrq_status kvrq_pages_add_seq(kvrq_pages* p, int64_t* seq_id) {
  if (!p || !seq_id) return set_error(KVRQ_EINVAL, "kvrq_pages_add_seq: NULL argument");
  std::lock_guard<std::mutex> lk(p->mu);
  return guarded("kvrq_pages_add_seq", [&] {
    alloc_check();
    p->seqs.emplace(p->next_id, kvrq_pages::Seq());  // the id is taken only once the entry exists
    *seq_id = p->next_id++;
    return KVRQ_OK;
  });
}

kvrq_status kvrq_pages_append(kvrq_pages* p, int64_t seq_id, int64_t n_tokens, int64_t* first_token) {
  if (!p || n_tokens < 0) return set_error(KVRQ_EINVAL, "kvrq_pages_append: bad arguments");
  std::lock_guard<std::mutex> lk(p->mu);
  auto it = p->seqs.find(seq_id);
  if (it == p->seqs.end()) return set_error(KVRQ_EINVAL, "kvrq_pages_append: unknown sequence");
  kvrq_pages::Seq& s = it->second;
  // tokens + n_tokens and its rounding up to whole pages must not overflow
  if (n_tokens > INT64_MAX - s.tokens - p->page_tokens)
    return set_error(KVRQ_EINVAL, "kvrq_pages_append: n_tokens too large (nothing appended)");
  const int64_t total = s.tokens + n_tokens;
  const int64_t need = (total + p->page_tokens - 1) / p->page_tokens - (int64_t)s.table.size();
  if (need > (int64_t)p->free_list.size())
    return set_error(KVRQ_EINVAL, "kvrq_pages_append: not enough free pages (nothing appended)");
  return guarded("kvrq_pages_append", [&] {
    if (need > 0) {
      alloc_check();
      s.table.reserve(s.table.size() + (size_t)need);  // may throw: nothing has moved yet
    }
    for (int64_t i = 0; i < need; ++i) {  // no allocation from here on
      s.table.push_back(p->free_list.back());
      p->free_list.pop_back();
    }
    if (first_token) *first_token = s.tokens;
    s.tokens = total;
    return KVRQ_OK;
  });
}

kvrq_status kvrq_pages_slots(kvrq_pages* p, int64_t seq_id, int64_t first, int64_t count, int64_t* slots) {
  if (!p || first < 0 || count < 0 || (count > 0 && !slots))
    return set_error(KVRQ_EINVAL, "kvrq_pages_slots: bad arguments");
  std::lock_guard<std::mutex> lk(p->mu);
  auto it = p->seqs.find(seq_id);
  if (it == p->seqs.end()) return set_error(KVRQ_EINVAL, "kvrq_pages_slots: unknown sequence");
  const kvrq_pages::Seq& s = it->second;
  // first <= tokens first, so that tokens - first cannot overflow and first + count is never formed
  if (first > s.tokens || count > s.tokens - first)
    return set_error(KVRQ_EINVAL, "kvrq_pages_slots: tokens past the sequence end");
  for (int64_t k = 0; k < count; ++k) {
    const int64_t t = first + k;
    slots[k] = (int64_t)s.table[(size_t)(t / p->page_tokens)] * p->page_tokens + t % p->page_tokens;
  }
  return KVRQ_OK;
}

kvrq_status kvrq_pages_block_table(kvrq_pages* p, int64_t seq_id, int32_t* pages, int64_t capacity,
                                   int64_t* n_pages, int64_t* n_tokens) {
  if (!p || capacity < 0 || (capacity > 0 && !pages)) return set_error(KVRQ_EINVAL, "kvrq_pages_block_table: bad arguments");
  std::lock_guard<std::mutex> lk(p->mu);
  auto it = p->seqs.find(seq_id);
  if (it == p->seqs.end()) return set_error(KVRQ_EINVAL, "kvrq_pages_block_table: unknown sequence");
  const kvrq_pages::Seq& s = it->second;
  if (n_pages) *n_pages = (int64_t)s.table.size();
  if (n_tokens) *n_tokens = s.tokens;
  if ((int64_t)s.table.size() > capacity) return set_error(KVRQ_EINVAL, "kvrq_pages_block_table: capacity too small");
  for (size_t i = 0; i < s.table.size(); ++i) pages[i] = s.table[i];
  return KVRQ_OK;
}

kvrq_status kvrq_pages_free_seq(kvrq_pages* p, int64_t seq_id) {
  if (!p) return set_error(KVRQ_EINVAL, "kvrq_pages_free_seq: NULL pool");
  std::lock_guard<std::mutex> lk(p->mu);
  auto it = p->seqs.find(seq_id);
  if (it == p->seqs.end()) return set_error(KVRQ_EINVAL, "kvrq_pages_free_seq: unknown sequence");
  // returned in reverse so that the sequence's first page is the next one handed out
  for (auto r = it->second.table.rbegin(); r != it->second.table.rend(); ++r) p->free_list.push_back(*r);
  p->seqs.erase(it);
  return KVRQ_OK;
}

kvrq_status kvrq_pages_stats(kvrq_pages* p, int64_t* free_pages, int64_t* n_seqs) {
  if (!p) return set_error(KVRQ_EINVAL, "kvrq_pages_stats: NULL pool");
  std::lock_guard<std::mutex> lk(p->mu);
  if (free_pages) *free_pages = (int64_t)p->free_list.size();
  if (n_seqs) *n_seqs = (int64_t)p->seqs.size();
  return KVRQ_OK;
}

}  // extern "C"

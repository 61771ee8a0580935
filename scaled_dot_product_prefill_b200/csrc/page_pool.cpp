// Host-side page pool for the paged KV cache: page allocation, reclaim and
// the per-sequence page tables that the attention kernels read.
//
// "Attention From Scratch" README, section "Paged KV Cache": fixed-size pages
// in one global pool, a page table per sequence, pages allocated as a
// sequence grows and reclaimed when it ends.  "LLM core technology", section
// "PagedAttention": a sequence's logical blocks map to non-contiguous
// physical blocks through that table, so no sequence needs contiguous memory
// and a finished sequence's pages serve the next one at once.
//
// The pool only manages page ids.  The K/V pools are device memory of the
// caller; the page table and lengths reach the device through
// attn_page_pool_upload, which copies the rows changed since the last upload.
#include <cuda_runtime_api.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "attn_b200.h"

// Plain C allocations only, so that the library needs no C++ runtime.
struct attn_page_pool {
  int num_pages, page_size, max_seqs, max_pages;
  int32_t* free_list;   // [num_pages] stack of free page ids; free_list[n_free - 1] is handed out next
  int n_free;
  int32_t* table;       // [max_seqs, max_pages], -1 after each sequence's last page
  int32_t* lens;        // [max_seqs] tokens per sequence
  int32_t* held;        // [max_seqs] pages per sequence
  int dirty_lo, dirty_hi;   // rows changed since the last upload: [lo, hi)
};

namespace {

int pages_for(long long tokens, int page_size) {
  return static_cast<int>((tokens + page_size - 1) / page_size);
}

void touch(attn_page_pool* p, int seq) {
  if (p->dirty_lo >= p->dirty_hi) {
    p->dirty_lo = seq;
    p->dirty_hi = seq + 1;
  } else {
    if (seq < p->dirty_lo) p->dirty_lo = seq;
    if (seq + 1 > p->dirty_hi) p->dirty_hi = seq + 1;
  }
}

}  // namespace

extern "C" {

void attn_page_pool_destroy(attn_page_pool_t* pool) {
  if (pool == nullptr) return;
  free(pool->free_list);
  free(pool->table);
  free(pool->lens);
  free(pool->held);
  free(pool);
}

attn_status_t attn_page_pool_create(int num_pages, int page_size, int max_seqs, int max_pages_per_seq,
                                    attn_page_pool_t** pool) {
  if (pool == nullptr) return ATTN_ERR_INVALID_ARG;
  *pool = nullptr;
  if (num_pages <= 0 || page_size <= 0 || max_seqs <= 0 || max_pages_per_seq <= 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_pages_per_seq) * page_size > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  attn_page_pool* p = static_cast<attn_page_pool*>(calloc(1, sizeof(attn_page_pool)));
  if (p == nullptr) return ATTN_ERR_INVALID_ARG;
  p->num_pages = num_pages;
  p->page_size = page_size;
  p->max_seqs = max_seqs;
  p->max_pages = max_pages_per_seq;
  const size_t cells = static_cast<size_t>(max_seqs) * max_pages_per_seq;
  p->free_list = static_cast<int32_t*>(malloc(sizeof(int32_t) * num_pages));
  p->table = static_cast<int32_t*>(malloc(sizeof(int32_t) * cells));
  p->lens = static_cast<int32_t*>(calloc(max_seqs, sizeof(int32_t)));
  p->held = static_cast<int32_t*>(calloc(max_seqs, sizeof(int32_t)));
  if (p->free_list == nullptr || p->table == nullptr || p->lens == nullptr || p->held == nullptr) {
    attn_page_pool_destroy(p);
    return ATTN_ERR_INVALID_ARG;
  }
  for (int i = 0; i < num_pages; ++i) p->free_list[i] = num_pages - 1 - i;   // page 0 is handed out first
  p->n_free = num_pages;
  for (size_t c = 0; c < cells; ++c) p->table[c] = -1;
  p->dirty_lo = 0;
  p->dirty_hi = max_seqs;   // the first upload writes every row
  *pool = p;
  return ATTN_OK;
}

attn_status_t attn_page_pool_resize(attn_page_pool_t* pool, int seq, int len) {
  if (pool == nullptr || seq < 0 || seq >= pool->max_seqs || len < 0) return ATTN_ERR_INVALID_ARG;
  const int want = pages_for(len, pool->page_size);
  if (want > pool->max_pages) return ATTN_ERR_INVALID_ARG;
  int32_t* row = pool->table + static_cast<size_t>(seq) * pool->max_pages;
  int have = pool->held[seq];
  if (want > have) {
    if (want - have > pool->n_free) return ATTN_ERR_OUT_OF_PAGES;
    for (; have < want; ++have) row[have] = pool->free_list[--pool->n_free];
  } else {
    // reclaim from the end of the sequence, so the page freed last is row[want]
    for (; have > want; --have) {
      pool->free_list[pool->n_free++] = row[have - 1];
      row[have - 1] = -1;
    }
  }
  pool->held[seq] = have;
  pool->lens[seq] = len;
  touch(pool, seq);
  return ATTN_OK;
}

attn_status_t attn_page_pool_release(attn_page_pool_t* pool, int seq) { return attn_page_pool_resize(pool, seq, 0); }

int attn_page_pool_free_pages(const attn_page_pool_t* pool) { return pool == nullptr ? -1 : pool->n_free; }

int attn_page_pool_seq_len(const attn_page_pool_t* pool, int seq) {
  if (pool == nullptr || seq < 0 || seq >= pool->max_seqs) return -1;
  return pool->lens[seq];
}

attn_status_t attn_page_pool_export(const attn_page_pool_t* pool, int32_t* page_table, int32_t* seq_lens) {
  if (pool == nullptr) return ATTN_ERR_INVALID_ARG;
  if (page_table != nullptr)
    memcpy(page_table, pool->table, sizeof(int32_t) * static_cast<size_t>(pool->max_seqs) * pool->max_pages);
  if (seq_lens != nullptr) memcpy(seq_lens, pool->lens, sizeof(int32_t) * pool->max_seqs);
  return ATTN_OK;
}

attn_status_t attn_page_pool_upload(attn_page_pool_t* pool, int32_t* page_table, int32_t* seq_lens,
                                    attn_stream_t stream) {
  if (pool == nullptr || page_table == nullptr || seq_lens == nullptr) return ATTN_ERR_INVALID_ARG;
  if (pool->dirty_lo >= pool->dirty_hi) return ATTN_OK;
  const size_t row = static_cast<size_t>(pool->max_pages);
  const size_t lo = pool->dirty_lo, n = pool->dirty_hi - pool->dirty_lo;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // pageable source: the runtime stages it before returning, so the pool may change afterwards
  if (cudaMemcpyAsync(page_table + lo * row, pool->table + lo * row, n * row * sizeof(int32_t),
                      cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(seq_lens + lo, pool->lens + lo, n * sizeof(int32_t), cudaMemcpyHostToDevice, s) !=
          cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  pool->dirty_lo = pool->dirty_hi = 0;
  return ATTN_OK;
}

}  // extern "C"

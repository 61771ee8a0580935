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

#include <algorithm>
#include <cstdint>
#include <new>
#include <vector>

#include "attn_b200.h"

struct attn_page_pool {
  int num_pages = 0, page_size = 0, max_seqs = 0, max_pages = 0;
  std::vector<int32_t> free_list;   // stack of free page ids; back() is handed out next
  std::vector<int32_t> table;       // [max_seqs, max_pages], -1 after each sequence's last page
  std::vector<int32_t> lens;        // [max_seqs] tokens per sequence
  std::vector<int32_t> held;        // [max_seqs] pages per sequence
  int dirty_lo = 0, dirty_hi = 0;   // rows changed since the last upload: [lo, hi)

  void touch(int seq) {
    if (dirty_lo >= dirty_hi) {
      dirty_lo = seq;
      dirty_hi = seq + 1;
    } else {
      dirty_lo = std::min(dirty_lo, seq);
      dirty_hi = std::max(dirty_hi, seq + 1);
    }
  }
};

namespace {

int pages_for(long long tokens, int page_size) {
  return static_cast<int>((tokens + page_size - 1) / page_size);
}

}  // namespace

extern "C" {

attn_status_t attn_page_pool_create(int num_pages, int page_size, int max_seqs, int max_pages_per_seq,
                                    attn_page_pool_t** pool) {
  if (pool == nullptr) return ATTN_ERR_INVALID_ARG;
  *pool = nullptr;
  if (num_pages <= 0 || page_size <= 0 || max_seqs <= 0 || max_pages_per_seq <= 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(max_pages_per_seq) * page_size > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  attn_page_pool* p = new (std::nothrow) attn_page_pool;
  if (p == nullptr) return ATTN_ERR_INVALID_ARG;
  try {
    p->num_pages = num_pages;
    p->page_size = page_size;
    p->max_seqs = max_seqs;
    p->max_pages = max_pages_per_seq;
    p->free_list.resize(num_pages);
    for (int i = 0; i < num_pages; ++i) p->free_list[i] = num_pages - 1 - i;   // page 0 first
    p->table.assign(static_cast<size_t>(max_seqs) * max_pages_per_seq, -1);
    p->lens.assign(max_seqs, 0);
    p->held.assign(max_seqs, 0);
  } catch (const std::bad_alloc&) {
    delete p;
    return ATTN_ERR_INVALID_ARG;
  }
  p->dirty_lo = 0;
  p->dirty_hi = max_seqs;   // the first upload writes every row
  *pool = p;
  return ATTN_OK;
}

void attn_page_pool_destroy(attn_page_pool_t* pool) { delete pool; }

attn_status_t attn_page_pool_resize(attn_page_pool_t* pool, int seq, int len) {
  if (pool == nullptr || seq < 0 || seq >= pool->max_seqs || len < 0) return ATTN_ERR_INVALID_ARG;
  const int want = pages_for(len, pool->page_size);
  if (want > pool->max_pages) return ATTN_ERR_INVALID_ARG;
  int32_t* row = pool->table.data() + static_cast<size_t>(seq) * pool->max_pages;
  int& have = pool->held[seq];
  if (want > have) {
    if (want - have > static_cast<int>(pool->free_list.size())) return ATTN_ERR_OUT_OF_PAGES;
    for (; have < want; ++have) {
      row[have] = pool->free_list.back();
      pool->free_list.pop_back();
    }
  } else {
    // reclaim from the end of the sequence, so the page freed last is row[want]
    for (; have > want; --have) {
      pool->free_list.push_back(row[have - 1]);
      row[have - 1] = -1;
    }
  }
  pool->lens[seq] = len;
  pool->touch(seq);
  return ATTN_OK;
}

attn_status_t attn_page_pool_release(attn_page_pool_t* pool, int seq) { return attn_page_pool_resize(pool, seq, 0); }

int attn_page_pool_free_pages(const attn_page_pool_t* pool) {
  return pool == nullptr ? -1 : static_cast<int>(pool->free_list.size());
}

int attn_page_pool_seq_len(const attn_page_pool_t* pool, int seq) {
  if (pool == nullptr || seq < 0 || seq >= pool->max_seqs) return -1;
  return pool->lens[seq];
}

attn_status_t attn_page_pool_export(const attn_page_pool_t* pool, int32_t* page_table, int32_t* seq_lens) {
  if (pool == nullptr) return ATTN_ERR_INVALID_ARG;
  if (page_table != nullptr) std::copy(pool->table.begin(), pool->table.end(), page_table);
  if (seq_lens != nullptr) std::copy(pool->lens.begin(), pool->lens.end(), seq_lens);
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
  if (cudaMemcpyAsync(page_table + lo * row, pool->table.data() + lo * row, n * row * sizeof(int32_t),
                      cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(seq_lens + lo, pool->lens.data() + lo, n * sizeof(int32_t), cudaMemcpyHostToDevice,
                      s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  pool->dirty_lo = pool->dirty_hi = 0;
  return ATTN_OK;
}

}  // extern "C"

// Host-side KV page allocator and admission planning (include/wmtp_pool.h).
//
// The pool is a stack of free page indices plus one allocated flag per page:
// alloc pops, release validates the whole list first and then pushes, so a
// bad release leaves the pool untouched.  Pages are uniform, so a free list
// cannot fragment.

#include <stdint.h>

#include <new>
#include <vector>

#include "wmtp_pool.h"

struct wmtp_page_pool {
  std::vector<int32_t> free_stack;  // free page indices; the top is handed out next
  std::vector<uint8_t> allocated;   // 1 while a page is held by a caller
};

extern "C" {

wmtp_status wmtp_pool_create(int32_t num_pages, wmtp_page_pool** pool) {
  if (pool == nullptr || num_pages < 1) return WMTP_ERR_INVALID_ARG;
  wmtp_page_pool* p = new (std::nothrow) wmtp_page_pool;
  if (p == nullptr) return WMTP_ERR_WORKSPACE;
  try {
    p->free_stack.resize(static_cast<size_t>(num_pages));
    p->allocated.assign(static_cast<size_t>(num_pages), 0);
  } catch (...) {
    delete p;
    return WMTP_ERR_WORKSPACE;
  }
  // lowest indices on top, so a fresh pool hands out 0, 1, 2, ...
  for (int32_t i = 0; i < num_pages; ++i) p->free_stack[static_cast<size_t>(i)] = num_pages - 1 - i;
  *pool = p;
  return WMTP_OK;
}

void wmtp_pool_destroy(wmtp_page_pool* pool) { delete pool; }

int32_t wmtp_pool_free_count(const wmtp_page_pool* pool) {
  return pool == nullptr ? 0 : static_cast<int32_t>(pool->free_stack.size());
}

wmtp_status wmtp_pool_alloc(wmtp_page_pool* pool, int32_t n, int32_t* pages) {
  if (pool == nullptr || n < 0 || (n > 0 && pages == nullptr)) return WMTP_ERR_INVALID_ARG;
  if (static_cast<size_t>(n) > pool->free_stack.size()) return WMTP_ERR_WORKSPACE;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t pg = pool->free_stack.back();
    pool->free_stack.pop_back();
    pool->allocated[static_cast<size_t>(pg)] = 1;
    pages[i] = pg;
  }
  return WMTP_OK;
}

wmtp_status wmtp_pool_release(wmtp_page_pool* pool, int32_t n, const int32_t* pages) {
  if (pool == nullptr || n < 0 || (n > 0 && pages == nullptr)) return WMTP_ERR_INVALID_ARG;
  const int64_t total = static_cast<int64_t>(pool->allocated.size());
  // validate everything first: in range, held, and listed once (the mark is
  // undone below whatever the outcome)
  bool ok = true;
  int32_t marked = 0;
  for (; marked < n; ++marked) {
    const int32_t pg = pages[marked];
    if (pg < 0 || pg >= total || pool->allocated[static_cast<size_t>(pg)] != 1) {
      ok = false;
      break;
    }
    pool->allocated[static_cast<size_t>(pg)] = 2;  // seen in this list
  }
  for (int32_t i = 0; i < marked; ++i) pool->allocated[static_cast<size_t>(pages[i])] = ok ? 0 : 1;
  if (!ok) return WMTP_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) pool->free_stack.push_back(pages[i]);
  return WMTP_OK;
}

wmtp_status wmtp_plan_admission(const wmtp_params* params, int64_t context, int32_t target_layers,
                                int32_t draft_layers, int32_t windowed, int64_t kv_budget_bytes,
                                wmtp_admission* out) {
  if (params == nullptr || out == nullptr || context < 0 || target_layers < 0 || draft_layers < 0 ||
      kv_budget_bytes < 0)
    return WMTP_ERR_INVALID_ARG;
  if (params->num_heads_kv <= 0 || params->head_dim <= 0 || params->page_size <= 0 || params->sinks < 0 ||
      params->window < 1 || params->gamma_max < 0)
    return WMTP_ERR_INVALID_ARG;
  const int64_t hkv = params->num_heads_kv;
  const int64_t d = params->head_dim;
  const int64_t tokens = context + params->gamma_max + 1;
  const int64_t pages = (tokens + params->page_size - 1) / params->page_size;
  const int64_t page_bytes = 2 * hkv * params->page_size * d * 2;  // K and V, bf16
  const int64_t layer_bytes = pages * page_bytes;
  const int64_t slots = static_cast<int64_t>(params->sinks) + params->window;
  const int64_t ring_bytes = 2 * slots * hkv * d * 2 + slots * 4 +                      // K, V, tags
                             2 * static_cast<int64_t>(params->gamma_max) * hkv * d * 2 +  // undo K, V
                             static_cast<int64_t>(params->gamma_max) * 4 + 2 * 4;       // undo tags, lengths
  out->pages_per_layer = pages;
  out->page_bytes = page_bytes;
  out->target_bytes = target_layers * layer_bytes;
  out->draft_bytes = draft_layers * (windowed ? ring_bytes : layer_bytes);
  out->bytes_per_request = out->target_bytes + out->draft_bytes;
  out->max_requests = out->bytes_per_request > 0 ? kv_budget_bytes / out->bytes_per_request : 0;
  return WMTP_OK;
}

}  // extern "C"

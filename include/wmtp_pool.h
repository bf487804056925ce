/*
 * wmtp_pool.h -- host-side KV page allocation and admission planning for
 * Windowed-MTP serving.
 *
 * Source: arxivlens view of "Windowed-MTP: Removing the Full-Context Draft-KV
 * Tax at Million-Token Context", Abstract and Results: once the draft reads
 * only a sink and a window, a compact ring buffer replaces the draft layer's
 * full KV pool, the freed pages return to the serving pool, and at 1M-token
 * context that room admits another concurrent request (the pages report
 * 7.7-11.1% of KV reclaimed).  The pages give no allocator; this one is a plain
 * free list over the page indices of one pool tensor (the `num_pages`
 * dimension of wmtp_paged_kv), so page tables built from it are valid inputs
 * of every wmtp_* attention call.
 *
 * Host memory only: nothing here touches a device.  Not thread-safe: callers
 * serialise access to one pool.
 */
#ifndef WMTP_POOL_H
#define WMTP_POOL_H

#include <stdint.h>

#include "wmtp.h"

#ifdef __cplusplus
extern "C" {
#endif

/* An allocator over page indices 0 .. num_pages-1. */
typedef struct wmtp_page_pool wmtp_page_pool;

/*
 * wmtp_pool_create -- a pool with every one of num_pages pages free.
 *   num_pages >= 1 (else WMTP_ERR_INVALID_ARG); *pool receives the handle,
 *   owned by the caller until wmtp_pool_destroy.
 */
wmtp_status wmtp_pool_create(int32_t num_pages, wmtp_page_pool** pool);

/* wmtp_pool_destroy -- release the handle (NULL is ignored). */
void wmtp_pool_destroy(wmtp_page_pool* pool);

/* wmtp_pool_free_count -- pages currently free (0 for NULL). */
int32_t wmtp_pool_free_count(const wmtp_page_pool* pool);

/*
 * wmtp_pool_alloc -- take n free pages, written to pages[0..n-1] (host
 * array).  All or nothing: with fewer than n pages free nothing is taken and
 * WMTP_ERR_WORKSPACE is returned.  n == 0 succeeds without writing.
 */
wmtp_status wmtp_pool_alloc(wmtp_page_pool* pool, int32_t n, int32_t* pages);

/*
 * wmtp_pool_release -- return n pages.  All or nothing: a page index outside
 * the pool, a page that is not allocated, or the same page twice in the list
 * returns WMTP_ERR_INVALID_ARG and releases nothing.
 */
wmtp_status wmtp_pool_release(wmtp_page_pool* pool, int32_t n, const int32_t* pages);

/* Per-request KV footprint and the number of requests one budget admits. */
typedef struct {
  int64_t pages_per_layer;    /* pages of one paged layer for one request */
  int64_t page_bytes;         /* K and V bytes of one page (all KV heads) */
  int64_t target_bytes;       /* the target layers' paged KV */
  int64_t draft_bytes;        /* native: the draft layers' paged KV; windowed: their rings */
  int64_t bytes_per_request;  /* target_bytes + draft_bytes */
  int64_t max_requests;       /* floor(kv_budget_bytes / bytes_per_request) */
} wmtp_admission;

/*
 * wmtp_plan_admission -- footprint of one request of `context` committed
 * tokens and the number of such requests a KV budget holds.
 *   Each paged layer of a request holds context + gamma_max + 1 tokens (the
 *   tokens a decode step appends before the rollback) in ceil(. / P) pages of
 *   Hkv x P x D bf16 for K and again for V.  target_layers layers are always
 *   paged.  With windowed == 0 the draft_layers are paged too; with
 *   windowed != 0 each keeps a ring instead: (S + W) slots of K and V, a tag
 *   per slot, an undo log of gamma_max entries (K, V, tag) and two lengths,
 *   the layout wmtp_ring describes.
 *   params: num_heads_kv, head_dim, page_size, sinks, window, gamma_max are
 *   read; context >= 0, target_layers >= 0, draft_layers >= 0,
 *   kv_budget_bytes >= 0, out != NULL (else WMTP_ERR_INVALID_ARG).
 */
wmtp_status wmtp_plan_admission(const wmtp_params* params, int64_t context, int32_t target_layers,
                                int32_t draft_layers, int32_t windowed, int64_t kv_budget_bytes,
                                wmtp_admission* out);

#ifdef __cplusplus
}
#endif

#endif /* WMTP_POOL_H */

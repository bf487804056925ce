/*
 * wmtp.h -- C ABI of libwmtp: the per-decode-step attention of Windowed-MTP
 * speculative decoding on one NVIDIA B200 (sm_100a).
 *
 * The method (from "Windowed-MTP: Removing the Full-Context Draft-KV Tax at
 * Million-Token Context", arxivlens paper view, Abstract): a built-in MTP
 * draft head runs gamma single-token decode attentions per decode step.  Run
 * natively, each one reads the draft layer's whole KV cache; Windowed-MTP
 * restricts the draft (only the draft) to S attention-sink tokens plus a
 * sliding window of the last W tokens, kept in a compact ring buffer.  The
 * target then verifies gamma+1 tokens with causal attention over its full
 * paged KV, so accepted tokens are unchanged.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument that is not a params/ring/kv descriptor is DEVICE
 *   memory owned by the caller.  Descriptor structs themselves are read on the
 *   host during the call and may be freed when it returns.  The library never
 *   allocates device memory.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream) and never synchronise the host.  The kernels of the
 *   attention calls, wmtp_ring_append and wmtp_paged_write are launched as
 *   programmatic dependents of the work before them on the stream: their
 *   launch and set-up may overlap its tail, but they touch no global memory
 *   before it has completed, so stream order holds for every input and
 *   output.  The calls
 *   can be captured in CUDA graphs (the first call on a device must come
 *   before any capture: it sets kernel attributes).
 * - Host-detectable argument errors return a negative wmtp_status before
 *   anything is launched.
 * - Device-detected problems (a page-table entry outside the pool, a length
 *   out of range, an inconsistent ring state) are OR-ed as WMTP_DEV_* bits
 *   into *status_word when status_word is non-NULL; the offending tile or
 *   sequence is skipped.  No kernel traps; every wait inside a kernel is
 *   bounded and reports WMTP_DEV_TIMEOUT if it gives up.
 * - bf16 means IEEE bfloat16 (raw 16-bit storage); fp32 accumulation.
 * - Supported shapes: head_dim in {64, 256}; num_heads_q / num_heads_kv = G
 *   with rows = num_q * G in 1..64, or in 1..128 for a verify of head_dim
 *   256 with num_q >= 2 (gamma = 8 with G = 8 is 72 rows); page_size in
 *   {16, 32, 64, 128, 256}; gamma_max <= 16; batch and num_heads_kv at most
 *   65535 (CUDA grid limits).  Anything else returns WMTP_ERR_UNSUPPORTED.
 *
 * Layouts
 * -------
 *   paged K or V pool : [num_pages][Hkv][page_size][D]      bf16
 *   page_table        : [batch][max_pages]                  int32
 *   kv_len            : [batch]                             int32
 *   draft query       : [batch][Hq][D]                      bf16
 *   verify query      : [batch][num_q][Hq][D]               bf16
 *   ring K or V       : [batch][Hkv][S+W][D]                bf16
 *   ring tags         : [batch][S+W]                        int32 (-1 = empty)
 *   undo K or V       : [batch][gamma_max][Hkv][D]          bf16
 *   output            : like the query, fp32 or bf16 (out_fp32)
 *   lse_out           : [batch][num_q][Hq] fp32, natural log (NULL = skip)
 *
 * Query head h reads KV head h / G (G = Hq / Hkv).
 */
#ifndef WMTP_H_
#define WMTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WMTP_OK = 0,
  WMTP_ERR_INVALID_ARG = -1, /* NULL where a pointer is required, bad size */
  WMTP_ERR_UNSUPPORTED = -2, /* a shape outside the supported set */
  WMTP_ERR_WORKSPACE = -3,   /* workspace too small or misaligned */
  WMTP_ERR_CUDA = -4         /* a CUDA runtime call failed (launch, attribute) */
} wmtp_status;

/* Bits the kernels OR into *status_word. */
#define WMTP_DEV_PAGE_OOB 0x1   /* page-table entry outside [0, num_pages) */
#define WMTP_DEV_LEN_OOB 0x2    /* kv_len < num_q or > max_pages * page_size */
#define WMTP_DEV_RING_STATE 0x4 /* ring len/committed inconsistent, or
                                   truncate_to outside [committed, len] */
#define WMTP_DEV_UNDO_FULL 0x8  /* speculative appends beyond gamma_max */
#define WMTP_DEV_TIMEOUT 0x10   /* a bounded in-kernel wait gave up */
#define WMTP_DEV_V_RANGE 0x20   /* reserved: no call sets it (the verify's value
                                   product takes V in bf16, at any magnitude) */

typedef struct {
  int32_t num_heads_q;  /* Hq */
  int32_t num_heads_kv; /* Hkv; Hq % Hkv == 0 */
  int32_t head_dim;     /* D */
  int32_t page_size;    /* P, tokens per page of the paged pools */
  int32_t sinks;        /* S, attention-sink tokens of the windowed draft */
  int32_t window;       /* W, sliding-window tokens of the windowed draft (>= 1) */
  int32_t gamma_max;    /* undo-log capacity: speculative appends per commit */
  float sm_scale;       /* softmax scale; 0 means 1/sqrt(D) */
} wmtp_params;

/* One attention layer's paged KV cache (all device pointers). */
typedef struct {
  void* k_pool;              /* [num_pages][Hkv][P][D] bf16 */
  void* v_pool;              /* [num_pages][Hkv][P][D] bf16 */
  int32_t num_pages;
  const int32_t* page_table; /* [batch][max_pages] */
  int32_t max_pages;
  const int32_t* kv_len;     /* [batch] valid tokens per sequence */
} wmtp_paged_kv;

/* Per-sequence compact draft ring buffers (all device pointers).  The ring
 * holds positions {0..min(S,len)-1} U {max(S,len-W)..len-1}; position p lives
 * in slot p if p < S, else S + (p - S) mod W. */
typedef struct {
  void* k;             /* [batch][Hkv][S+W][D] bf16 */
  void* v;             /* [batch][Hkv][S+W][D] bf16 */
  int32_t* tags;       /* [batch][S+W] position held by each slot, -1 = empty */
  int32_t* len;        /* [batch] positions appended (speculative included) */
  int32_t* committed;  /* [batch] length at the last commit */
  void* undo_k;        /* [batch][gamma_max][Hkv][D] bf16, overwritten entries */
  void* undo_v;        /* [batch][gamma_max][Hkv][D] bf16 */
  int32_t* undo_tags;  /* [batch][gamma_max] tags of the overwritten entries */
  int32_t batch;
} wmtp_ring;

/* Status as a static string ("ok", "invalid argument", ...). */
const char* wmtp_status_string(int32_t status);

/* Library version as "major.minor.patch". */
const char* wmtp_version(void);

/*
 * wmtp_draft_attn_full -- native MTP draft attention.
 * Source: arxivlens view of the paper, Abstract (the draft head attends over
 * the full KV cache in each of its gamma forwards); howtospark case study
 * "Does speculative decode still pay at 128K context?", Background.
 *
 * For every sequence b and query head h: o = softmax(sm_scale * K q) V over
 * positions 0 .. kv_len[b]-1 of the draft layer's paged cache (kv_len
 * includes the token appended for this draft step).
 *   q        : [batch][Hq][D] bf16
 *   kv       : the draft layer's paged cache
 *   out      : [batch][Hq][D], fp32 if out_fp32 else bf16
 *   lse_out  : [batch][Hq] fp32 or NULL.
 *   kv_len[b] == 0 is an empty sequence: o = 0, lse = -inf.  A kv_len below
 *   num_q or above max_pages * page_size sets WMTP_DEV_LEN_OOB and is treated
 *   as empty.
 *   workspace: device scratch for split-KV partials, 256-byte aligned.  Call
 *              with workspace == NULL to get the size in *workspace_bytes
 *              (nothing is launched).  The size depends on the device's SM
 *              count, batch, shapes and max_pages.
 */
wmtp_status wmtp_draft_attn_full(const wmtp_params* params, int32_t batch, const void* q,
                                 const wmtp_paged_kv* kv, void* out, int32_t out_fp32,
                                 float* lse_out, void* workspace, size_t* workspace_bytes,
                                 int32_t* status_word, void* stream);

/*
 * wmtp_draft_attn_windowed_paged -- Windowed-MTP draft attention read through
 * the page table, with no ring.
 * Source: arxivlens view, Abstract (the draft attends a sink plus a sliding
 * window); the same attended set as wmtp_draft_attn_windowed, for callers that
 * keep the draft layer's full paged cache.  The window may change from call
 * to call (params->window), which a fixed-capacity ring cannot follow.
 *
 * For every sequence b and query head h: o = softmax(sm_scale * K q) V over
 * positions p < min(S, kv_len[b]) and max(S, kv_len[b] - W) <= p < kv_len[b]
 * of the paged cache.  Only the pages holding those positions are read: at
 * most ceil(S/64) + ceil(W/64) + 1 tiles of 64 tokens per sequence.
 *   Arguments, layouts, workspace and errors as wmtp_draft_attn_full;
 *   params->sinks >= 0 and params->window >= 1 (else WMTP_ERR_INVALID_ARG).
 */
wmtp_status wmtp_draft_attn_windowed_paged(const wmtp_params* params, int32_t batch, const void* q,
                                           const wmtp_paged_kv* kv, void* out, int32_t out_fp32,
                                           float* lse_out, void* workspace, size_t* workspace_bytes,
                                           int32_t* status_word, void* stream);

/*
 * wmtp_draft_attn_windowed -- Windowed-MTP draft attention over the ring.
 * Source: arxivlens view, Abstract (StreamingLLM-style sink plus window on the
 * draft only; the compact ring buffer); readpriors post "Your Million-Token
 * Pipeline Is Bleeding Speed ...", What happened.
 *
 * For every sequence b and head h: o = softmax(sm_scale * K q) V over the ring
 * entries whose tag t satisfies t < min(S, len[b]) or
 * max(S, len[b] - W) <= t < len[b].  Reads at most S+W entries per sequence,
 * whatever the context length.
 *   q: [ring->batch][Hq][D] bf16; out / lse_out / workspace as above.
 */
wmtp_status wmtp_draft_attn_windowed(const wmtp_params* params, const void* q,
                                     const wmtp_ring* ring, void* out, int32_t out_fp32,
                                     float* lse_out, void* workspace, size_t* workspace_bytes,
                                     int32_t* status_word, void* stream);

/*
 * wmtp_ring_append -- append draft K/V to the rings, with speculative undo.
 * Source: arxivlens view, Abstract and Technical contributions (a compact
 * ring buffer holding only the sink and window entries).  The undo log is
 * this library's reading of how a speculative draft token that the target
 * rejects is taken back out of the ring (the pages do not say).
 *
 * Per sequence b, in order:
 *   1. if truncate_to != NULL and truncate_to[b] >= 0: roll back to length
 *      truncate_to[b] (must lie in [committed[b], len[b]]), restoring the
 *      entries the rolled-back speculative appends overwrote, newest first;
 *   2. append n_new[b] tokens (k_new/v_new rows 0..n_new[b]-1) at positions
 *      len[b] .. len[b]+n_new[b]-1.  If speculative, each append first saves
 *      the entry it overwrites to the undo log (at most gamma_max since the
 *      last commit); otherwise only the tokens that survive in the final
 *      sink + window are written;
 *   3. if !speculative: commit (committed[b] = len[b]; undo log emptied).
 *   k_new, v_new: [batch][max_new][Hkv][D] bf16; n_new: [batch], each in
 *   [0, max_new]; n_new may be NULL when max_new == 0.
 * Results are bit-exact copies of the given bf16 values.
 */
wmtp_status wmtp_ring_append(const wmtp_params* params, const wmtp_ring* ring,
                             const int32_t* truncate_to, const int32_t* n_new,
                             const void* k_new, const void* v_new, int32_t max_new,
                             int32_t speculative, int32_t* status_word, void* stream);

/*
 * wmtp_ring_reset -- empty every ring: tags = -1, K/V and undo zeroed,
 * len = committed = 0.  Call once before first use.
 */
wmtp_status wmtp_ring_reset(const wmtp_params* params, const wmtp_ring* ring, void* stream);

/*
 * wmtp_verify_attn -- target verify attention of num_q = gamma+1 queries.
 * Source: arxivlens view, Abstract (verification keeps full-context attention,
 * so the target distribution is preserved); howtospark case study, Method (one
 * cycle = gamma draft forwards plus one batched verify).
 *
 * Query i (0 <= i < num_q) of sequence b sits at position kv_len[b]-num_q+i
 * and attends causally to positions 0 .. kv_len[b]-num_q+i of the layer's
 * paged cache; the caller has already written the num_q new tokens' K/V.
 * All G query heads of a KV head and all num_q queries are processed together
 * so each K/V byte is read once.
 *   q: [batch][num_q][Hq][D] bf16; out: [batch][num_q][Hq][D];
 *   lse_out: [batch][num_q][Hq]; workspace as for wmtp_draft_attn_full.
 */
wmtp_status wmtp_verify_attn(const wmtp_params* params, int32_t batch, int32_t num_q,
                             const void* q, const wmtp_paged_kv* kv, void* out,
                             int32_t out_fp32, float* lse_out, void* workspace,
                             size_t* workspace_bytes, int32_t* status_word, void* stream);

/*
 * wmtp_verify_attn_append -- wmtp_paged_write of the num_q new tokens at
 * positions kv_len[b]-num_q .. kv_len[b]-1, then wmtp_verify_attn, in one
 * call.  Source: howtospark case study, Method (a verify layer appends its
 * gamma+1 tokens and attends over them); the fusion is this library's.
 * On the tcgen05 verify path (head_dim 256, 2 <= num_q, 9..128 rows per KV
 * head) the verify kernel writes each new row itself, with plain stores
 * ordered before the bulk copy that loads its tile, so no separate write is
 * launched; other shapes launch the paged write in front of the verify.
 *   k_new, v_new: [batch][num_q][Hkv][D] bf16, 16-byte aligned, not NULL
 *   when workspace is given.  Pages and lengths are checked as in
 *   wmtp_paged_write (a new row on a page outside the pool is not written and
 *   sets WMTP_DEV_PAGE_OOB).  Everything else as wmtp_verify_attn.
 */
wmtp_status wmtp_verify_attn_append(const wmtp_params* params, int32_t batch, int32_t num_q, const void* q,
                                    const void* k_new, const void* v_new, const wmtp_paged_kv* kv, void* out,
                                    int32_t out_fp32, float* lse_out, void* workspace, size_t* workspace_bytes,
                                    int32_t* status_word, void* stream);

/*
 * wmtp_verify_attn_slice -- verify attention over one slice of each
 * sequence's context (context parallelism).
 * Not on the pages as such: the pages verify on one GPU.  A sequence whose
 * context is spread over several caches (one per GPU, each holding a
 * contiguous range of positions) is verified by calling this on every slice
 * and merging the (out, lse) pairs with wmtp_splitkv_combine, which is exact
 * because softmax attention over a union of disjoint key sets is the
 * log-sum-exp merge of the attentions over each set.
 *
 * As wmtp_verify_attn, except that query i of sequence b attends the
 * positions p < kv_len[b] of this cache with p <= q_pos0[b] + i, where
 * q_pos0[b] (device int32, required) is the position of query 0 counted from
 * the slice's first token: for a slice starting at global position s of a
 * sequence whose num_q queries sit at n - num_q .. n - 1, q_pos0 = n - num_q - s.
 * A slice entirely before the queries (q_pos0 >= kv_len) is attended in
 * full; a query that sees no position of the slice gets out = 0, lse = -inf.
 * kv_len[b] may be smaller than num_q.
 */
wmtp_status wmtp_verify_attn_slice(const wmtp_params* params, int32_t batch, int32_t num_q, const void* q,
                                   const wmtp_paged_kv* kv, const int32_t* q_pos0, void* out, int32_t out_fp32,
                                   float* lse_out, void* workspace, size_t* workspace_bytes, int32_t* status_word,
                                   void* stream);

/*
 * wmtp_splitkv_combine -- merge split-KV partial attention results.
 * Not on the pages: the standard log-sum-exp identity behind split-KV
 * (flash-decoding) decode attention, needed to spread one sequence over the
 * GPU's SMs.  For each row r:
 *   m = max_s lse[r][s];  w_s = exp(lse[r][s] - m);
 *   out[r] = sum_s w_s part_o[r][s] / sum_s w_s;  lse_out[r] = m + log sum_s w_s.
 * Splits with lse = -inf carry no weight; a row whose splits are all empty
 * gives out = 0, lse = -inf.
 *   part_o: [rows][nsplit][head_dim] fp32; part_lse: [rows][nsplit] fp32
 *   out: [rows][head_dim] fp32 or bf16; lse_out: [rows] or NULL.
 */
wmtp_status wmtp_splitkv_combine(int32_t rows, int32_t head_dim, int32_t nsplit,
                                 const float* part_o, const float* part_lse, void* out,
                                 int32_t out_fp32, float* lse_out, void* stream);

/*
 * wmtp_paged_write -- write new tokens' K/V into a paged cache.
 * Support call (the append half of a decode step: the draft writes one token
 * per draft forward, a verify layer writes its gamma+1 tokens).  For each
 * sequence b and j < n_new: position pos0[b]+j goes to page
 * page_table[b][(pos0[b]+j)/P], row (pos0[b]+j)%P.  kv->kv_len is not read or
 * changed.
 *   pos0: [batch] int32; k_new, v_new: [batch][n_new][Hkv][D] bf16.
 */
wmtp_status wmtp_paged_write(const wmtp_params* params, int32_t batch, const wmtp_paged_kv* kv,
                             const int32_t* pos0, int32_t n_new, const void* k_new,
                             const void* v_new, int32_t* status_word, void* stream);

/*
 * wmtp_draft_attn_full_noalloc -- wmtp_draft_attn_full without a workspace.
 * The paper has no counterpart to this call; it exists for callers that
 * cannot allocate device memory for the split-KV scratch: runtimes that plan
 * all device memory before serving starts and forbid later allocations, and
 * plugin hosts whose kernel interface passes only inputs and outputs.
 *
 * Same arguments, semantics and results as wmtp_draft_attn_full, minus the
 * workspace pair.  The partial results go to one fixed device array of
 * WMTP_NOALLOC_SCRATCH_BYTES inside the library; every GPU that loads the
 * library holds that array until the process exits.  The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current; a failed lookup is retried by the
 *     next call).  Make that first call before any stream capture.
 *   - The array's device memory is claimed when the library's GPU code is
 *     loaded on a device.  With CUDA's default lazy module loading that is the
 *     first call of this library on that device, whichever entry point it is.
 *     A caller that must have all device memory claimed before a given point
 *     makes one call per device before it (or sets CUDA_MODULE_LOADING=EAGER,
 *     which loads the code when the CUDA context is created).
 *   - A call whose scratch would exceed WMTP_NOALLOC_SCRATCH_BYTES returns
 *     WMTP_ERR_WORKSPACE and launches nothing (the size is the one that
 *     wmtp_draft_attn_full reports in *workspace_bytes).
 *   - All calls share the array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero: every call overwrites each
 *     partial it reads.  Calls that overlap on the GPU (different streams,
 *     no ordering between them) race on the array and give wrong results.
 */
#define WMTP_NOALLOC_SCRATCH_BYTES (4u << 20)
wmtp_status wmtp_draft_attn_full_noalloc(const wmtp_params* params, int32_t batch, const void* q,
                                         const wmtp_paged_kv* kv, void* out, int32_t out_fp32,
                                         float* lse_out, int32_t* status_word, void* stream);

/*
 * wmtp_selftest_wait -- run the bounded in-kernel wait on its own.
 * The paper has no counterpart to this call, and it is not on the attention
 * path.  It lets a test check on a live GPU that a wait which never completes
 * gives up, reports WMTP_DEV_TIMEOUT, and leaves the context usable.
 *
 * One thread initialises a shared-memory mbarrier that expects one arrival.
 * It then waits for the barrier's first phase, with the same bounded wait
 * every attention kernel uses: it gives up after WMTP_WAIT_LIMIT_CYCLES SM
 * clocks, about 2 s at 1.9 GHz.
 *   arrive != 0 : the thread arrives first, so the wait returns at once and
 *                 no bit is set.
 *   arrive == 0 : nothing arrives.  The wait gives up at the limit and
 *                 WMTP_DEV_TIMEOUT is OR-ed into *status_word.
 *   status_word : device int32, NULL = skip.
 *   cycles_out  : device int64, NULL = skip.  Receives the SM clocks the wait
 *                 took.
 * A misaligned pointer returns WMTP_ERR_INVALID_ARG; a failed launch returns
 * WMTP_ERR_CUDA.  Asynchronous on `stream` like every other call.
 */
#define WMTP_WAIT_LIMIT_CYCLES 4000000000LL
wmtp_status wmtp_selftest_wait(int32_t arrive, int32_t* status_word, int64_t* cycles_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WMTP_H_ */

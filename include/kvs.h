/*
 * kvs.h -- C ABI of libkvs: host-streamed paged quantized KV attention on one
 * NVIDIA B200 (sm_100a).
 *
 * The method (sources: "RaymondHuang210129/llama.cpp-adaptive-kv-streaming",
 * Summary; "llama.cpp adaptive KV streaming - spec fork notes", Phase arena and
 * Configuration; "Feature/adaptive kv stream integration", PR #326):
 *   - the full KV history of every layer lives in pinned host memory and is
 *     authoritative; K is stored as Q8_0 and V as Q4_0 (blocks of 32 values,
 *     fp16 scale; the other V types are listed at kvs_config.type_v), grouped
 *     in 256-token pages;
 *   - per layer only the most recent R pages are resident in device memory;
 *     older pages stream in order through one device ring of N page slots that
 *     all layers share, on a copy stream, so the copy of page i+k overlaps
 *     attention over page i;
 *   - attention is exact over every page (streaming on == streaming off).
 *
 * Conventions for every call below:
 *   - return 0 (KVS_OK) on success or a negative KVS_E_* code; on failure the
 *     handle is unchanged and kvs_last_error() describes the cause;
 *   - device pointers are plain CUDA device addresses (for example a torch
 *     tensor's data_ptr()); kvs_append/kvs_attend also accept host pointers and
 *     then stage them through library-owned device buffers on `stream`;
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     stream ordered and asynchronous: results are valid once `stream` has
 *     completed.  Appends and attends of one handle must be issued on one
 *     stream, or the caller orders its streams itself;
 *   - the library owns the pinned host history, the device arena (resident
 *     pages, ring slots, split partials, staging), its copy stream and events.
 *     The caller owns Q/K/V/out/lse buffers and `stream`.
 *   - there is no CPU fallback: without a usable CUDA device kvs_create fails.
 */
#ifndef KVS_H
#define KVS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define KVS_OK         0
#define KVS_E_INVAL   (-1) /* bad argument, shape or unsupported K/V type pair   */
#define KVS_E_ARENA   (-2) /* arena smaller than one page or than its contents   */
#define KVS_E_WIDTH   (-3) /* n_q > max_q_tokens ("decode batch too wide")        */
#define KVS_E_ORDER   (-4) /* append not contiguous / attend beyond the history  */
#define KVS_E_CUDA    (-5) /* a CUDA runtime call failed                          */
#define KVS_E_TIMEOUT (-6) /* a bounded host wait gave up                         */
#define KVS_E_NOMEM   (-7) /* host (pinned) allocation failed                     */

/* ---- cache types: K Q8_0 with V F16, Q4_0, Q4_1, Q5_0, Q5_1 or Q8_0; or the
 *      f16-f16 pair (K and V both F16) ------------------------------------- */
#define KVS_TYPE_F16  1
#define KVS_TYPE_Q4_0 2
#define KVS_TYPE_Q4_1 3
#define KVS_TYPE_Q5_0 6
#define KVS_TYPE_Q5_1 7
#define KVS_TYPE_Q8_0 8

/* ---- page kinds reported by kvs_page_location --------------------------- */
#define KVS_PAGE_ABSENT   (-1)
#define KVS_PAGE_RESIDENT 1
#define KVS_PAGE_STREAMED 2

/* ---- flags --------------------------------------------------------------- */
/* Record CUDA events around every kernel (kvs_get_stats).  Profiling runs all
 * kernels on the caller's stream, one after another, so that the events time
 * one kernel each; steps are slower than without it. */
#define KVS_FLAG_PROFILE 1
/* Set by config resolution when the handle runs a phase arena (arena_bytes
 * with n_resident_pages = 0); a resolved config passed back keeps it. */
#define KVS_FLAG_PHASE_ARENA 2

typedef struct kvs_config {
    int n_layers;         /* attention layers sharing the pool, auxiliary layers included (e.g. 16+1) */
    int n_q_heads;        /* query heads; a multiple of n_kv_heads */
    int n_kv_heads;       /* KV heads; q head h reads kv head h / (n_q_heads/n_kv_heads) */
    int head_dim;         /* must be 128 */
    int page_tokens;      /* must be 256 */
    int max_ctx;          /* host history capacity in tokens per layer */
    int n_resident_pages; /* resident pages per layer; 0 = auto: with arena_bytes = 0, 10 % of
                             max_ctx (8-page floor, 8192 MiB ceiling over all layers); with a
                             fixed arena_bytes, the most pages that fit beside the ring, the
                             split partials and the staging (at most pages(max_ctx)) */
    int n_ring_slots;     /* device ring slots (pages); 0 = all-resident mode, which needs
                             n_resident_pages >= pages(max_ctx) */
    int max_q_tokens;     /* widest append / attend batch (1, 1+n_draft or a 256-token ubatch) */
    int type_k;           /* KVS_TYPE_Q8_0, or KVS_TYPE_F16 together with type_v = KVS_TYPE_F16:
                             the f16-f16 pair, which the flash-attention build always compiles
                             ("llama.cpp adaptive KV streaming - spec fork notes", TLDR); its
                             page head is 131,072 B (K values fp16 [256 tok][128 dims], then V
                             values the same way, no scales) */
    int type_v;           /* KVS_TYPE_Q4_0 (page head 53,248 B), KVS_TYPE_Q8_0 (69,632 B: V codes
                             stored like K's; the q8_0/q8_0 pair of the "Feature/adaptive kv
                             stream integration" pull request's runs), or one of the other
                             legal cache types of the flash-attention build ("llama.cpp
                             adaptive KV streaming - spec fork notes", TLDR):
                             KVS_TYPE_Q5_0 (57,344 B: Q4_0's nibbles plus a word of fifth
                             bits per block), KVS_TYPE_Q4_1 (55,296 B: Q4_0's layout plus an
                             fp16 block minimum m, x = d q + m), KVS_TYPE_Q5_1 (59,392 B:
                             Q5_0's layout plus m), KVS_TYPE_F16 (100,352 B: the V values
                             as fp16 [256 tok][128 dims], no scales) */
    int chunk_pages;      /* pages per H2D copy; 0 = auto (n_ring_slots/2); must divide n_ring_slots */
    int flags;            /* KVS_FLAG_* */
    int zero_copy_pct;    /* 0..100: share of each layer's streamed pages (the newest ones) that
                             decode calls (n_q * n_q_heads/n_kv_heads <= 8) read in place from
                             the mapped pinned history by the SMs, over PCIe, while the copy
                             engine brings the older ones through the ring.  In-place reads pay
                             no per-copy cost; the ring can copy ahead into the next layer.
                             100 = no ring copies for decode (the design the "Feature/adaptive
                             kv stream integration" pull request's review found in its
                             kernels).  Wider calls take zero_copy_pct_wide instead; a ring
                             is still required when pages stream. */
    size_t arena_bytes;   /* device arena budget; 0 = exact fit; else must hold one page and all
                             resident pages + ring + partials + staging (KVS_E_ARENA if not).
                             With n_resident_pages = 0 the handle runs a phase arena: it
                             allocates exactly arena_bytes and lends it to the current phase
                             (kvs_set_phase), with a pinned region at its top (below) */
    int n_aux_layers;     /* phase arena only: the last n_aux_layers layers are auxiliary (a
                             speculative draft's attention layer, e.g. MTP): their resident pages
                             live in the pinned region at the arena top, they stream the rest
                             through the shared ring, and kvs_draft_eject returns their bytes to
                             the pool; 0 = none */
    int aux_resident_pages; /* resident pages per auxiliary layer (in the pinned region); 0 = the
                             10 % rule of the target layers */
    int zero_copy_pct_wide; /* 0..100: the in-place share, as zero_copy_pct, for calls wider than
                             decode (verify batches, prefill chunks: the tensor-core kernel),
                             whose in-place launch reads its pages over PCIe with 16-byte
                             asynchronous copies; 0 = those calls stream through the ring only */
} kvs_config;

/* ---- phase arena ------------------------------------------------------------
 * "RaymondHuang210129/llama.cpp-adaptive-kv-streaming", Summary: one bounded
 * device allocation is lent to either prefill or decode, never both; "llama.cpp
 * adaptive KV streaming - spec fork notes", Phase arena and New arena and
 * context API: the decode layout is re-reserved at the verify width, a pinned
 * region is bump-allocated from the arena top (the draft's KV and weights) with
 * the compute region below it, and the draft-active decode pool is what
 * remains after the pin and the phase compute slab.
 * Layout from the bottom: error word, resident pages of the target layers
 * (R per layer), ring, compute slab (split partials and staging for the
 * phase's width), free bytes; from the top: the auxiliary layers' resident
 * pages, then kvs_pin reservations. */
#define KVS_PHASE_PREFILL 0
#define KVS_PHASE_DECODE  1

typedef struct kvs_arena_status {
    int phase;               /* KVS_PHASE_PREFILL or KVS_PHASE_DECODE */
    int width;               /* widest append / attend batch of the phase */
    int n_resident_pages;    /* resident pages per target layer */
    int aux_resident_pages;  /* resident pages per auxiliary layer; 0 while the draft is ejected */
    int draft_active;        /* 1 unless kvs_draft_eject released the pinned region */
    int phase_arena;         /* 1 when the handle runs a phase arena */
    size_t arena_bytes;      /* the allocation */
    size_t compute_bytes;    /* split partials + staging + error word of the phase */
    size_t resident_bytes;   /* target layers' resident pages */
    size_t ring_bytes;
    size_t aux_bytes;        /* auxiliary layers' resident pages (pinned, at the top) */
    size_t pinned_bytes;     /* kvs_pin reservations (below the auxiliary pages) */
    size_t free_bytes;       /* arena_bytes minus everything above */
} kvs_arena_status;

typedef struct kvs_stats {
    uint64_t appends, attends;         /* calls */
    uint64_t tokens_appended;
    uint64_t pages_streamed;           /* pages copied host -> ring */
    uint64_t bytes_h2d;                /* ring copy bytes */
    uint64_t bytes_resident_read;      /* resident page bytes attended */
    uint64_t h2d_copies;               /* cudaMemcpyAsync calls issued for the ring */
    uint64_t kernel_launches;          /* kernels launched by the library */
    /* filled when KVS_FLAG_PROFILE is set: summed CUDA-event durations, ms
     * (decode_zc: the launches that read streamed pages in place over PCIe) */
    double ms_decode_resident, ms_decode_ring, ms_merge, ms_append, ms_chunk_mma, ms_decode_zc;
    uint64_t n_decode_resident, n_decode_ring, n_merge, n_append, n_chunk_mma, n_decode_zc;
    uint64_t bytes_decode_resident, bytes_decode_ring, bytes_decode_zc; /* page bytes read */
    /* the tensor-core kernel's launches that read streamed pages in place */
    double ms_chunk_zc;
    uint64_t n_chunk_zc, bytes_chunk_zc;
} kvs_stats;

typedef struct kvs_s kvs_t;

/* ---- pure host functions (no GPU needed) -------------------------------- */

/* Validate `in` and fill `out` with every automatic field resolved
 * (n_resident_pages, chunk_pages, arena_bytes = bytes actually needed).
 * `host_bytes` (optional) receives the pinned history size.  The gates follow
 * PR #326's configuration validation (type pair, single page byte size) and its
 * minimum stage of one page ("Diagnostic log"). */
int kvs_resolve_config(const kvs_config* in, kvs_config* out, size_t* host_bytes);

/* Bytes of one page of one layer (all kv heads, K + V): 256 * n_kv * 1664/8. */
size_t kvs_page_bytes(const kvs_config* cfg);

/* Where page `page` of a layer holding n_tokens tokens lives: *kind is
 * KVS_PAGE_RESIDENT (*index = resident slot = page mod R), KVS_PAGE_STREAMED
 * (*index = streaming ordinal = page; pages 0..S-1 stream in ascending order)
 * or KVS_PAGE_ABSENT.  The R most recent pages are resident. */
int kvs_plan_page(const kvs_config* resolved, int n_tokens, int page, int* kind, int* index);

/* The ring schedule of one kvs_attend call of n_q query tokens whose streamed
 * pages 0..s_ring-1 go through the transfer ring ("RaymondHuang210129/
 * llama.cpp-adaptive-kv-streaming", Summary: one shared ring buffer), with the
 * handle's ring counter at ring_ctr0: the host-to-device copies in order, copy
 * i moving pages page0[i] .. page0[i]+pages[i]-1 into ring slots slot0[i] ..
 * slot0[i]+pages[i]-1.  One copy per chunk_pages pages, each into the next
 * group of chunk_pages slots; on the tensor-core path with more than one
 * 128-row tile per kv head, the last chunk goes as two pieces into one group
 * (the first (5p + 7) / 8 of its p pages, then the rest).  Writes at most
 * max_copies entries (the arrays may be NULL when max_copies is 0) and returns
 * the number of copies, or KVS_E_INVAL for a null config, n_q < 1, a negative
 * s_ring, ring_ctr0 or max_copies, or an unresolved ring (slots without a
 * chunk size).  Pure host logic: no device is touched. */
int kvs_plan_ring(const kvs_config* resolved, int n_q, int s_ring, long long ring_ctr0, int* page0, int* pages,
                  int* slot0, int max_copies);

/* ---- draft eject controller (pure host) ------------------------------------
 * The dynamic draft eject of "llama.cpp adaptive KV streaming - spec fork
 * notes" (Dynamic draft eject; Results): a pinned draft (an MTP block and its
 * KV, or a DFlash2 draft) borrows part of the arena; the controller ejects it
 * when the target's decode working set outgrows the eject threshold and
 * re-enables it when the working set fits again, with hysteresis and a
 * stability count.  The library runs no draft model: a serving loop calls
 * kvs_eject_step once per decode batch and acts on the transitions. */
typedef struct kvs_eject_params {
    int keep_pages;      /* eject threshold, in 256-token pages per layer of the target's decode
                            working set; 0 = capacity_pages (eject at streaming onset) */
    int reenable_pages;  /* re-enable once the working set is this many pages below the
                            threshold; 0 = default 8 */
    int stable_decodes;  /* consecutive decode batches a transition condition must hold;
                            0 = default 4 */
    int capacity_pages;  /* draft-active decode capacity: resident pages per layer the arena
                            holds with the draft pinned (kvs_draft_capacity_pages) */
} kvs_eject_params;

typedef struct kvs_eject_state {
    int draft_active;    /* 1 while the draft is active */
    int streak;          /* consecutive batches for which the transition condition held */
} kvs_eject_state;

/* Fill the defaults of zero fields of *p and start with the draft active.
 * KVS_E_INVAL for null pointers, negative fields or a zero threshold. */
int kvs_eject_init(kvs_eject_params* p, kvs_eject_state* s);

/* One decode batch whose target working set is `working_pages` pages per
 * layer.  Active: the draft is ejected after stable_decodes consecutive
 * batches above the threshold.  Ejected: it is re-enabled after
 * stable_decodes consecutive batches at or below threshold - reenable_pages.
 * A batch that breaks the condition resets the streak.  Returns 1 when the
 * state changed (*s tells which way), 0 when not, KVS_E_INVAL on bad input. */
int kvs_eject_step(const kvs_eject_params* p, kvs_eject_state* s, int working_pages);

/* The draft-active decode capacity: the most resident pages per layer that
 * fit in the config's arena (arena_bytes > 0) once `pinned_bytes` are
 * reserved for the draft ("what remains of the arena after the pinned
 * reservation and the phase compute slab").  KVS_E_ARENA if none fit. */
int kvs_draft_capacity_pages(const kvs_config* cfg, size_t pinned_bytes, int* pages);

/* ---- handle lifecycle ----------------------------------------------------- */

/* Allocate the pinned host history (n_layers * pages(max_ctx) pages, mapped
 * into the device address space) and the device arena on `device`, create the
 * copy stream and ring events.  All-or-nothing: on failure nothing is leaked
 * and *out is NULL. */
int kvs_create(const kvs_config* cfg, int device, kvs_t** out);

/* Wait (bounded by timeout_s, polling) for the library's copy stream and the
 * given stream, then free everything.  NULL is a no-op. */
void kvs_destroy(kvs_t* kv);

/* ---- hot path ------------------------------------------------------------- */

/* Quantize n_tok new K/V rows (fp16, layout [n_tok][n_kv_heads][head_dim]) of
 * `layer` at positions pos0..pos0+n_tok-1: K -> Q8_0, V -> Q4_0.  The blocks
 * are written to the host history and, for pages that are resident after the
 * append, to their resident slot.  pos0 must be <= the layer's length (pos0 <
 * length rolls the history back to pos0 first, as a rejected speculative draft
 * does); pos0 + n_tok <= max_ctx; n_tok >= 1.  Device K/V may be of any width
 * (history pre-fill); host K/V are staged and limited to max_q_tokens (else
 * KVS_E_WIDTH).  Pages that re-enter the resident set on a roll-back are copied
 * back from the host history on `stream`. */
int kvs_append(kvs_t* kv, int layer, int pos0, int n_tok, const void* k_f16,
               const void* v_f16, void* stream);

/* Attention of n_q query tokens (fp16, [n_q][n_q_heads][head_dim]) at
 * positions pos0..pos0+n_q-1 over the layer's quantized history: query j sees
 * keys 0..pos0+j.  Needs pos0+n_q <= length and n_q <= max_q_tokens
 * (KVS_E_WIDTH).  Writes out (fp32 [n_q][n_q_heads][head_dim]) and lse (fp32
 * [n_q][n_q_heads], natural log of sum(exp(q.k/sqrt(head_dim)))); lse may be
 * NULL.  Resident pages are attended in place; streamed pages are copied
 * through the ring on the library's copy stream and attended as they land;
 * per-split partials are merged by log-sum-exp.  Device buffers must suit the
 * kernels' vector accesses (KVS_E_INVAL otherwise): q 8-byte aligned for
 * decode widths (n_q * n_q_heads/n_kv_heads <= 8) and 16-byte aligned for
 * wider calls; out 16-byte aligned when n_q * n_q_heads >= 1024, else 4-byte;
 * lse 4-byte.  Host buffers have no alignment requirement. */
int kvs_attend(kvs_t* kv, int layer, int pos0, int n_q, const void* q_f16, float* out,
               float* lse, void* stream);

/* ---- diagnostics ---------------------------------------------------------- */

/* Copy page `page` of `layer` to host_dst in canonical block layout:
 * [256 tokens][n_kv_heads][head_dim/32] Q8_0 blocks of 34 bytes (fp16 d, 32 x
 * int8), then [256][n_kv_heads][head_dim/32] V blocks: Q4_0 blocks of 18
 * bytes (fp16 d, byte j = q_j | q_(j+16) << 4), Q8_0 blocks of 34 bytes when
 * type_v is KVS_TYPE_Q8_0, or Q5_0 blocks of 22 bytes when it is KVS_TYPE_Q5_0
 * (fp16 d, a little-endian word whose bit j is bit 4 of q_j, then 16 bytes
 * holding the low 4 bits as Q4_0 does); Q4_1 (20 bytes) and Q5_1 (24 bytes)
 * blocks put the fp16 block minimum m right after d; F16 blocks are the 32
 * fp16 values (64 bytes); with type_k = KVS_TYPE_F16 the K blocks are the 32
 * fp16 values too (64 bytes).  from_device = 0 reads the host history,
 * 1 reads the resident slot (KVS_E_INVAL if the page is not resident).  The
 * caller must have synchronized the streams that wrote the page. */
int kvs_export_page(kvs_t* kv, int layer, int page, int from_device, void* host_dst);

/* kvs_plan_page for the layer's current length. */
int kvs_page_location(kvs_t* kv, int layer, int page, int* kind, int* index);

/* Current length (tokens) of a layer's history. */
int kvs_layer_length(kvs_t* kv, int layer, int* n_tokens);

/* The resolved configuration of a handle. */
int kvs_get_config(kvs_t* kv, kvs_config* out);

/* Counters; with KVS_FLAG_PROFILE, first waits (bounded) for recorded events
 * and folds their durations in.  kvs_reset_stats zeroes them. */
int kvs_get_stats(kvs_t* kv, kvs_stats* out);
int kvs_reset_stats(kvs_t* kv);

/* Change the in-place shares of streamed pages (kvs_config zero_copy_pct for
 * decode calls and zero_copy_pct_wide for wider calls, 0..100; -1 leaves a
 * share as it is) for later calls, e.g. to compare the copy-engine ring alone
 * (0) with in-place reads alone (100) on one handle.  The split partials are
 * sized for every share at kvs_create.  KVS_E_INVAL outside -1..100.  A CUDA
 * graph captured earlier keeps the shares it was captured with. */
int kvs_set_zero_copy_pct(kvs_t* kv, int pct, int pct_wide);

/* Pure host: the layout a phase arena (resolved config with a budget and
 * auto resident pages) takes for a phase of the given width (1..max_q_tokens)
 * with `pinned_bytes` of kvs_pin reservations and the draft active or
 * ejected.  KVS_E_ARENA if no resident page fits; KVS_E_INVAL if the config
 * is not a phase arena. */
int kvs_phase_layout(const kvs_config* resolved, int width, size_t pinned_bytes, int draft_active,
                     kvs_arena_status* out);

/* Re-lend the arena to a phase: KVS_PHASE_PREFILL takes width max_q_tokens,
 * KVS_PHASE_DECODE takes `width` (1 + n_draft; 0 = 1).  Waits (bounded) for
 * the handle's work, lays the arena out for the phase (a narrower compute slab
 * leaves room for more resident pages) and copies the pages that are resident
 * in the new layout from the authoritative host history on `stream`.  Later
 * calls wider than the phase's width fail with KVS_E_WIDTH ("phase arena decode
 * batch too wide").  CUDA graphs captured before the switch are invalid after
 * it.  KVS_E_INVAL if the handle has no phase arena. */
int kvs_set_phase(kvs_t* kv, int phase, int width, void* stream);

/* Bump-allocate `bytes` (rounded up to 256) from the top of the arena, below
 * the auxiliary layers' pages and earlier reservations, for a draft's weights
 * or state; the target's resident set shrinks if it must (pages copied as in
 * kvs_set_phase, on `stream`).  *dev_ptr = the reservation's device address.
 * KVS_E_ARENA if the current phase would keep no resident page; KVS_E_INVAL
 * while the draft is ejected or without a phase arena. */
int kvs_pin(kvs_t* kv, size_t bytes, void** dev_ptr, void* stream);

/* Draft eject: release the whole pinned region (the auxiliary layers' pages
 * and every kvs_pin reservation) to the target's resident pages; appends and
 * attends on auxiliary layers fail with KVS_E_INVAL until kvs_draft_restore.
 * Restore re-reserves the auxiliary pages at the top (the target shrinks back)
 * and copies them from the host history, which stayed authoritative.  Both
 * are no-ops when already in that state. */
int kvs_draft_eject(kvs_t* kv, void* stream);
int kvs_draft_restore(kvs_t* kv, void* stream);

/* The arena layout in use. */
int kvs_get_arena(kvs_t* kv, kvs_arena_status* out);

/* Turn KVS_FLAG_PROFILE on (1) or off (0) for later calls. */
int kvs_set_profiling(kvs_t* kv, int enable);

/* Bounded host wait for all work the library enqueued (copy stream) and for
 * `stream`: polls, returns KVS_E_TIMEOUT after timeout_s seconds. */
int kvs_sync(kvs_t* kv, void* stream, double timeout_s);

/* Measure pinned host->device copy bandwidth with `chunk_bytes` per
 * cudaMemcpyAsync over `total_bytes` (best of `reps`), using the library's own
 * copy stream and a scratch region of the device arena.  GB/s in *gbs. */
int kvs_measure_h2d(kvs_t* kv, size_t chunk_bytes, size_t total_bytes, int reps, double* gbs);

/* Attention over caller-owned device pages that allocates nothing.
 *
 * The paper has no counterpart to this call.  It serves callers that cannot
 * allocate device memory on their hot path: an engine whose own pool owns all
 * device memory, a server whose allocations are frozen after start-up so no
 * request can fail for memory, or a latency-critical loop that must avoid
 * cudaMalloc's implicit device synchronization.  It needs no handle: the
 * split partials live in one static device array inside libkvs (2 MiB + 32 KiB
 * per GPU that loads the library, held until exit); nothing is allocated.
 *
 * pages: device, 16-byte aligned, n_pages pages in libkvs's page layout, page
 *        p = tokens [256p, 256p+256): [n_kv_heads][53,248-byte page head] with
 *        the page head = Kq int8 [256][128] | Kd fp16 [256][4] |
 *        Vq u8 [256][4][16] (byte j: code j low nibble, code j+16 high) |
 *        Vd fp16 [256][4];
 * keys 0..n_tokens-1 are attended; query j sits at pos0+j and sees keys
 * 0..pos0+j; q fp16 [n_q][n_q_heads][128]; out fp32 [n_q][n_q_heads][128];
 * lse fp32 [n_q][n_q_heads] or NULL.  Limit: n_q * n_q_heads <= 64, else
 * KVS_E_WIDTH.  Alignment (KVS_E_INVAL otherwise): pages 16 bytes, q 8 bytes,
 * out and lse 4 bytes.  If a bounded wait inside the kernels gives up (the
 * GPU stalled for over a second), out and lse come back as NaN.  The first call on a device looks up the static array's device
 * address (with that device current); make that first call before any stream
 * capture.  Every call shares the array, so calls whose kernels may overlap on
 * the GPU race: order them on one stream.  Stream ordered and asynchronous. */
int kvs_attend_pages_static(const void* pages, int n_pages, int n_tokens, int n_q_heads,
                            int n_kv_heads, int pos0, int n_q, const void* q_f16, float* out,
                            float* lse, void* stream);

/* Failure-detection self-test: launch one GPU thread that waits, through the
 * same bounded mbarrier wait every libkvs kernel uses, on a barrier phase that
 * nothing completes.  The wait gives up after limit_s seconds (0 < limit_s <=
 * 10) and records KVS_ERR_WAIT_TIMEOUT in the error word, which is returned in
 * *err_bits; the device stays usable.  Needs no handle. */
#define KVS_ERR_WAIT_TIMEOUT 1
int kvs_selftest_bounded_wait(int device, double limit_s, int* err_bits);

/* Last error text of the handle (or of the calling thread's last failed
 * kvs_create / pure call when kv is NULL). */
const char* kvs_last_error(kvs_t* kv);

#ifdef __cplusplus
}
#endif
#endif /* KVS_H */

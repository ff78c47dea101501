// kvs_runtime.cpp -- host runtime behind the C ABI in include/kvs.h: config
// validation and auto sizing (10 % rule, or the resident fit of a fixed
// arena), the pinned host history, the device arena (resident pages, ring
// slots, split partials, staging), the page table, the copy-engine ring with
// its events, the share of streamed pages decode reads in place from the
// mapped history, the call sequencing of append/attend over the caller's
// stream and four library streams, and the draft eject controller.
//
// Method sources:
//  * "RaymondHuang210129/llama.cpp-adaptive-kv-streaming", Summary: the full KV
//    history stays in pinned system RAM, only resident pages plus one shared
//    ring buffer occupy device memory, an auxiliary layer borrows the same pool.
//  * "llama.cpp adaptive KV streaming - spec fork notes", Phase arena:
//    speculative verify batches: a generation batch wider than the configured
//    maximum fails ("decode batch too wide") -> KVS_E_WIDTH.
//  * "Feature/adaptive kv stream integration" (PR #326): auto sizing (10 % of
//    the context resident per layer, 2048-token floor, 8192 MiB ceiling), the
//    configuration gates (supported K/V type pair, one page byte size for all
//    streamed layers), the minimum stage of one page, and the review's
//    observation that a real implementation needs a device staging pool, a
//    page table and a cudaMemcpyAsync ring (its own kernels read mapped host
//    memory directly: the in-place share keeps that design as an option).
//  * "llama.cpp adaptive KV streaming - spec fork notes", Dynamic draft eject:
//    the eject threshold, re-enable band and stability count.
#include <algorithm>
#include <chrono>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include "../../include/kvs.h"
#include "kvs_internal.h"

using namespace kvs;

namespace {

thread_local std::string g_last_error;

constexpr size_t kAlign = 256;
size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

std::string fmt(const char* f, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, f);
    vsnprintf(buf, sizeof buf, f, ap);
    va_end(ap);
    return buf;
}

long pages_for(long tokens) { return (tokens + kPageTokens - 1) / kPageTokens; }

// Auto resident pages: 10 % of max_ctx per layer rounded up to whole pages,
// 2048-token floor, 8192 MiB ceiling over all layers.
long auto_resident(long max_ctx, size_t page_bytes, int n_layers) {
    long pages = (max_ctx + 10L * kPageTokens - 1) / (10L * kPageTokens);
    pages = std::max(pages, (2048L + kPageTokens - 1) / kPageTokens);
    const long cap = (long)((8192ull << 20) / (page_bytes * (size_t)n_layers));
    pages = std::min(pages, cap);
    return std::max(pages, 1L);
}

// Split layout, in half-page stages per split.
//  * decode kernel (<= 8 query rows per kv head, warp-level mma.sync): resident
//    splits sized so the resident launch has about two CTAs per SM, one stage
//    per split inside a ring chunk so a chunk's kernel spreads over many SMs;
//    decode batches wider than 64 rows in all: at most 8 resident splits and
//    one split per ring chunk, which keeps the partial buffer and merge small.
//  * tcgen05 kernel (more rows per kv head: verify batches, prefill chunks):
//    one CTA per SM; resident splits chosen for the fewest waves x stages, and
//    per ring chunk as many splits as fit one wave beside the other units.
constexpr int kSmallRows = 64;
constexpr int kTargetCtas = 296;  // 148 SMs x 2 resident CTAs
constexpr int kMaxDecodeRows = 8;

bool use_tcgen05(const kvs_config& c, int n_q) { return n_q * (c.n_q_heads / c.n_kv_heads) > kMaxDecodeRows; }
bool wide_regime(const kvs_config& c, int n_q) { return n_q * c.n_q_heads > kSmallRows; }
int m_tiles(const kvs_config& c, int n_q) { return (n_q * (c.n_q_heads / c.n_kv_heads) + 127) / 128; }
// CTAs per kv head and split of the tcgen05 kernel: one per pair of M tiles
int tile_pairs(const kvs_config& c, int n_q) { return (m_tiles(c, n_q) + 1) / 2; }

// tcgen05 path: splits sized for about one CTA per SM per ring chunk and
// about two waves over the resident pages (the kernel holds one CTA per SM).
constexpr int kSms = 148;

// Splits of the resident launch and of one ring-chunk launch (each split is an
// equal share of the launch's half-page stages).
constexpr long kResCtaStages = 4;  // raw stages per resident CTA beside ring launches
constexpr long kResSplitsMax = 16; // splits per such resident launch, at most

int res_splits(const kvs_config& c, long R_eff, int n_q, bool ring) {
    const long stages = 2 * R_eff;
    if (use_tcgen05(c, n_q)) {
        // one CTA per SM: pick the split count that minimizes waves x stages
        // per split on a full machine (ties -> fewer splits, fewer partials)
        const long units = (long)c.n_kv_heads * tile_pairs(c, n_q);
        long best = 1, best_cost = -1;
        for (long sp = 1; sp <= std::min(stages, 32L); ++sp) {
            const long cost = ((units * sp + kSms - 1) / kSms) * ((stages + sp - 1) / sp);
            if (best_cost < 0 || cost < best_cost) { best = sp; best_cost = cost; }
        }
        // Beside ring-chunk launches the resident pages go in a sequence of
        // launches of short CTAs (kResCtaStages raw stages each) that fold
        // into one set of records: a CTA holds its SM until it ends, and a
        // ring chunk whose copy has landed must not wait behind a long
        // resident CTA.  A launch is about one wave (3 splits for the 40 units
        // of a 256-token prefill chunk, 16 for the 8 of a verify batch).
        if (ring) return (int)std::min<long>(stages, std::max(1L, std::min(kResSplitsMax, (long)kSms / units)));
        return (int)best;
    }
    if (wide_regime(c, n_q)) return (int)std::min(stages, 8L);
    // decode kernel: one wave of two CTAs per SM
    const long per_split = (long)c.n_kv_heads * ((n_q * (c.n_q_heads / c.n_kv_heads) + 7) / 8);
    return (int)std::min(stages, std::max(1L, (long)kTargetCtas / per_split));
}

// One copy of a call's ring schedule: streamed pages [page0, page0 + pages)
// into ring slots [slot0, slot0 + pages).  new_group: the copy starts a ring
// group (and waits for that group's previous launch); otherwise it continues
// the group of the copy before it.
struct RingCopy {
    long page0;
    int pages;
    int slot0;
    bool new_group;
};

// The ring schedule of one call whose streamed pages [0, S_ring) go through
// the ring, in ascending page order: one copy per chunk_pages pages, each into
// the next group (ring_ctr0, ring_ctr0 + 1, ... mod the group count).  Wide
// tensor-core calls (more than one M tile) send the last chunk as two pieces
// into the slots of one group: the first (5 p + 7) / 8 of its p pages, then
// the rest.  The launch after the final copy, which nothing overlaps, then
// attends fewer pages; only the first piece waits for the group to be free.
// (On B200 a launch costs about 14 us plus 2.7 us per page and an 8-page copy
// 65.5 us: a first piece of 5/8 is the largest whose launch ends before the
// second piece's copy.)  Returns the groups used (the ring counter's advance).
long plan_ring(const kvs_config& c, int n_q, long S_ring, long long ring_ctr0, std::vector<RingCopy>& out) {
    out.clear();
    const int chunk = c.chunk_pages;
    const long n_groups = chunk > 0 ? c.n_ring_slots / chunk : 0;
    if (S_ring <= 0 || n_groups <= 0) return 0;
    const bool split_tail = use_tcgen05(c, n_q) && m_tiles(c, n_q) > 1 && chunk >= 2;
    const long last0 = (S_ring - 1) / chunk * chunk;  // first page of the last chunk
    long groups = 0;
    int gidx = 0, slot_off = 0, cpages = 0;
    for (long i0 = 0; i0 < S_ring; i0 += cpages) {
        cpages = (int)std::min<long>(chunk, S_ring - i0);
        const bool piece = split_tail && i0 >= last0;
        if (piece && i0 == last0 && cpages >= 2) cpages = (5 * cpages + 7) / 8;
        const bool fresh = !piece || i0 == last0;
        if (fresh) {
            gidx = (int)((ring_ctr0 + groups) % n_groups);
            ++groups;
            slot_off = 0;
        }
        out.push_back(RingCopy{i0, cpages, gidx * chunk + slot_off, fresh});
        slot_off += cpages;
    }
    return groups;
}

int ring_splits(const kvs_config& c, int n_q, int chunk_pages) {
    const int stages = 2 * chunk_pages;
    if (use_tcgen05(c, n_q)) {
        // at most one wave, leaving SMs to the resident launch when a chunk's
        // units cannot fill the machine twice
        const int units = c.n_kv_heads * tile_pairs(c, n_q);
        return std::min(stages, std::max(1, kSms / units));
    }
    return wide_regime(c, n_q) ? 1 : stages;
}

// Zero-copy decode: the last zero_copy_pct % of a layer's streamed pages (the
// ones nearest the resident window) are read in place by one launch, about one
// CTA per SM (the resident and ring launches share the SMs); the ring brings
// the older ones.
// Calls on the tensor-core path take the wide share; their in-place launch
// keeps to about kZcTcCtas CTAs (one per SM), leaving SMs to the resident and
// ring launches beside it.
constexpr int kZcTcCtas = 120;
long zero_copy_pages(const kvs_config& c, int n_q, long S) {
    const int pct = use_tcgen05(c, n_q) ? c.zero_copy_pct_wide : c.zero_copy_pct;
    if (pct <= 0) return 0;
    return std::min(S, (S * pct + 50) / 100);
}
int zc_splits(const kvs_config& c, long S_zc, int n_q) {
    if (use_tcgen05(c, n_q)) {
        const long units = (long)c.n_kv_heads * tile_pairs(c, n_q);
        return (int)std::min(2 * S_zc, std::max(1L, (long)kZcTcCtas / units));
    }
    const long per_split = (long)c.n_kv_heads * ((n_q * (c.n_q_heads / c.n_kv_heads) + 7) / 8);
    return (int)std::min(2 * S_zc, std::max(1L, (long)kSms / per_split));
}

long count_splits(const kvs_config& c, int n_q, long R_eff, long S) {
    const long S_zc = zero_copy_pages(c, n_q, S), S_ring = S - S_zc;
    long n = res_splits(c, R_eff, n_q, S_ring > 0 && c.chunk_pages > 0);
    if (S_zc > 0) n += zc_splits(c, S_zc, n_q);
    if (S_ring > 0 && c.chunk_pages > 0) {
        const long full = S_ring / c.chunk_pages, tail = S_ring % c.chunk_pages;
        if (use_tcgen05(c, n_q)) {
            // the tensor-core ring launches merge into one set of records (the
            // first chunk, the widest, writes them; later chunks accumulate)
            n += ring_splits(c, n_q, full > 0 ? c.chunk_pages : (int)tail);
        } else {
            n += full * ring_splits(c, n_q, c.chunk_pages);
            if (tail) n += ring_splits(c, n_q, (int)tail);
        }
    }
    return n;
}

// capacity of the partial buffer in (split x row) records: the largest need
// over every query width the handle accepts, at the longest history (split
// counts only grow with the number of resident and streamed pages), and over
// every in-place share, so that kvs_set_zero_copy_pct can change it later
size_t partial_records_r(const kvs_config& c, long R) {
    const long P = pages_for(c.max_ctx);
    const long R_eff = std::min<long>(R, P);
    const long S = c.n_ring_slots > 0 ? P - R_eff : 0;
    size_t best = 1;
    for (int n_q = 1; n_q <= c.max_q_tokens; ++n_q) {
        kvs_config cz = c;
        const bool tc = use_tcgen05(c, n_q);
        // decode widths: every share; wider calls: ring only, in place only, and
        // both together bound the counts (the in-place and ring launches have
        // fixed split counts there)
        const int shares = tc ? 3 : 101;
        for (int k = 0; k < shares; ++k) {
            if (tc) cz.zero_copy_pct_wide = k * 50;
            else cz.zero_copy_pct = k;
            best = std::max(best, (size_t)count_splits(cz, n_q, R_eff, S) * (size_t)(n_q * c.n_q_heads));
        }
    }
    return best;
}
// over the target layers' and the auxiliary layers' resident counts
size_t partial_records(const kvs_config& c) {
    size_t n = partial_records_r(c, c.n_resident_pages);
    if (c.n_aux_layers > 0) n = std::max(n, partial_records_r(c, std::max(1, c.aux_resident_pages)));
    return n;
}

// the layers whose resident pages sit in the main resident region
int target_layers(const kvs_config& c) { return c.n_layers - c.n_aux_layers; }

// bytes of the auxiliary layers' resident pages (pinned at the arena top)
size_t aux_region_bytes(const kvs_config& c) {
    const size_t pb = (size_t)c.n_kv_heads * page_head_bytes(c.type_v, c.type_k);
    return align_up((size_t)c.n_aux_layers * c.aux_resident_pages * pb, 1024);
}

// Layout of the arena's lower part: resident pages of the target layers, ring,
// split partials and staging for the widest batch (max_q_tokens), error word.
struct ArenaLayout {
    size_t resident, ring, part_ml, part_acc, stage_q, stage_kv, stage_out, stage_lse, err, total;
};

ArenaLayout arena_layout(const kvs_config& c) {
    const size_t pb = (size_t)c.n_kv_heads * page_head_bytes(c.type_v, c.type_k);
    const size_t rows = (size_t)c.max_q_tokens * c.n_q_heads;
    const size_t recs = partial_records(c);
    ArenaLayout L{};
    size_t off = 0;
    L.resident = off; off = align_up(off + (size_t)target_layers(c) * c.n_resident_pages * pb, 1024);
    L.ring = off;     off = align_up(off + (size_t)c.n_ring_slots * pb, 1024);
    L.part_ml = off;  off = align_up(off + recs * sizeof(float2));
    L.part_acc = off; off = align_up(off + recs * kHeadDim * sizeof(float));
    L.stage_q = off;  off = align_up(off + rows * kHeadDim * sizeof(__half));
    L.stage_kv = off; off = align_up(off + 2 * (size_t)c.max_q_tokens * c.n_kv_heads * kHeadDim * sizeof(__half));
    L.stage_out = off; off = align_up(off + rows * kHeadDim * sizeof(float));
    L.stage_lse = off; off = align_up(off + rows * sizeof(float));
    L.err = off;      off = align_up(off + 256);
    L.total = off;
    return L;
}

ArenaLayout arena_layout_with(kvs_config c, long resident_pages) {
    c.n_resident_pages = (int)resident_pages;
    return arena_layout(c);
}

// the most resident pages per layer (at most P) whose arena fits in `budget`
// bytes, 0 if none does.  The arena is not monotone in the resident count:
// fewer resident pages mean more streamed chunks and so more split partials,
// so the counts are tried from P down.
long resident_fit(const kvs_config& c, size_t budget, long P) {
    const size_t per_page = (size_t)target_layers(c) * c.n_kv_heads * page_head_bytes(c.type_v, c.type_k);
    const long top = std::min<long>(std::max(1L, P), (long)(budget / per_page));  // resident bytes alone
    for (long r = top; r >= 1; --r)
        if (arena_layout_with(c, r).total <= budget) return r;
    return 0;
}

int resolve(const kvs_config* in, kvs_config* out, size_t* host_bytes, std::string& why) {
    if (!in || !out) { why = "null config"; return KVS_E_INVAL; }
    kvs_config c = *in;
    if (c.n_layers < 1) { why = "n_layers must be >= 1"; return KVS_E_INVAL; }
    if (c.n_kv_heads < 1 || c.n_q_heads < 1 || c.n_q_heads % c.n_kv_heads != 0) {
        why = fmt("n_q_heads (%d) must be a positive multiple of n_kv_heads (%d)", c.n_q_heads, c.n_kv_heads);
        return KVS_E_INVAL;
    }
    if (c.head_dim != kHeadDim) { why = fmt("head_dim %d unsupported (only 128)", c.head_dim); return KVS_E_INVAL; }
    if (c.page_tokens != kPageTokens) { why = fmt("page_tokens %d unsupported (only 256)", c.page_tokens); return KVS_E_INVAL; }
    if (!kv_pair_supported(c.type_k, c.type_v)) {
        why = "block KV streaming is not supported for this K/V cache type pair "
              "(K=Q8_0 with V=F16, Q4_0, Q4_1, Q5_0, Q5_1 or Q8_0; or K=F16 with V=F16)";
        return KVS_E_INVAL;
    }
    if (c.max_ctx < 1) { why = "max_ctx must be >= 1"; return KVS_E_INVAL; }
    if (c.max_q_tokens < 1 || c.max_q_tokens > 4096) { why = "max_q_tokens must be in [1, 4096]"; return KVS_E_INVAL; }
    if (c.n_resident_pages < 0 || c.n_ring_slots < 0 || c.chunk_pages < 0) {
        why = "negative page counts";
        return KVS_E_INVAL;
    }
    if (c.zero_copy_pct < 0 || c.zero_copy_pct > 100 || c.zero_copy_pct_wide < 0 || c.zero_copy_pct_wide > 100) {
        why = fmt("zero_copy_pct %d / zero_copy_pct_wide %d outside 0..100", c.zero_copy_pct, c.zero_copy_pct_wide);
        return KVS_E_INVAL;
    }
    // a phase arena: a fixed budget with the resident set fitted to it (a
    // resolved phase-arena config carries the flag and is re-fitted)
    const bool phase = c.arena_bytes != 0 && (c.n_resident_pages == 0 || (c.flags & KVS_FLAG_PHASE_ARENA));
    if (phase) c.n_resident_pages = 0;
    if (c.n_aux_layers < 0 || c.n_aux_layers >= c.n_layers || c.aux_resident_pages < 0) {
        why = fmt("n_aux_layers (%d) must be in [0, n_layers) and aux_resident_pages >= 0", c.n_aux_layers);
        return KVS_E_INVAL;
    }
    if ((c.n_aux_layers > 0 || c.aux_resident_pages > 0) && !phase) {
        why = "auxiliary layers need a phase arena (arena_bytes with n_resident_pages = 0)";
        return KVS_E_INVAL;
    }
    const size_t pb = (size_t)c.n_kv_heads * page_head_bytes(c.type_v, c.type_k);
    const long P = pages_for(c.max_ctx);
    if (c.n_ring_slots == 0) {
        c.chunk_pages = 0;
    } else {
        if (c.chunk_pages == 0) c.chunk_pages = std::max(1, c.n_ring_slots / 2);
        if (c.chunk_pages > c.n_ring_slots || c.n_ring_slots % c.chunk_pages != 0) {
            why = fmt("chunk_pages (%d) must divide n_ring_slots (%d)", c.chunk_pages, c.n_ring_slots);
            return KVS_E_INVAL;
        }
    }
    if (c.arena_bytes != 0 && c.arena_bytes < pb) {
        why = fmt("arena %zu B is below the minimum stage of one page (%zu B)", c.arena_bytes, pb);
        return KVS_E_ARENA;
    }
    size_t aux_bytes = 0;
    if (c.n_resident_pages == 0) {
        if (c.arena_bytes == 0) {
            c.n_resident_pages = (int)auto_resident(c.max_ctx, pb, c.n_layers);
        } else {
            // a fixed arena: the auxiliary layers' pages are pinned at its top;
            // the target's resident pages get what the pin, the ring, the split
            // partials and the staging leave (the decode KV grant of the arena)
            if (c.n_aux_layers > 0) {
                c.aux_resident_pages = (int)std::min<long>(
                    P, c.aux_resident_pages > 0 ? c.aux_resident_pages : auto_resident(c.max_ctx, pb, c.n_aux_layers));
                aux_bytes = aux_region_bytes(c);
            }
            const long fit = aux_bytes < c.arena_bytes ? resident_fit(c, c.arena_bytes - aux_bytes, P) : 0;
            if (fit < 1) {
                why = fmt("arena %zu B cannot hold any resident set besides ring + partials (%zu B with one page)"
                          " and the auxiliary layers' %zu B",
                          c.arena_bytes, arena_layout_with(c, 1).total, aux_bytes);
                return KVS_E_ARENA;
            }
            c.n_resident_pages = (int)fit;
        }
    }
    if (c.n_resident_pages > P) c.n_resident_pages = (int)P;
    if (c.n_ring_slots == 0 && c.n_resident_pages < P) {
        why = fmt("all-resident mode (n_ring_slots=0) needs n_resident_pages >= %ld", P);
        return KVS_E_INVAL;
    }
    const ArenaLayout L = arena_layout(c);
    if (c.arena_bytes != 0) {
        if (c.arena_bytes < L.total + aux_bytes) {
            why = fmt("arena %zu B cannot hold resident pages + ring + partials (%zu B)", c.arena_bytes,
                      L.total + aux_bytes);
            return KVS_E_ARENA;
        }
    }
    // a phase arena keeps its budget: the whole allocation, re-lent by phase
    if (phase) c.flags |= KVS_FLAG_PHASE_ARENA;
    else c.arena_bytes = L.total;
    if (host_bytes) *host_bytes = (size_t)c.n_layers * (size_t)P * pb;
    *out = c;
    return KVS_OK;
}

int plan_page_r(long R, long n_tokens, long page, int* kind, int* index) {
    const long P = pages_for(n_tokens);
    if (page < 0 || page >= P) {
        *kind = KVS_PAGE_ABSENT;
        *index = -1;
        return KVS_OK;
    }
    if (page >= P - R) {
        *kind = KVS_PAGE_RESIDENT;
        *index = (int)(page % R);
    } else {
        *kind = KVS_PAGE_STREAMED;
        *index = (int)page;
    }
    return KVS_OK;
}
int plan_page(const kvs_config& c, long n_tokens, long page, int* kind, int* index) {
    return plan_page_r(c.n_resident_pages, n_tokens, page, kind, index);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// device alias of a pinned (page-locked) host buffer when it is 16-byte
// aligned; nullptr for pageable host memory, device memory or misalignment.
// Small inputs and outputs in pinned memory then cross PCIe inside the
// library's kernels instead of queueing on the copy engines behind the ring.
const void* pinned_alias16(const void* p) {
    cudaPointerAttributes at;
    if (!p || cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
    return (reinterpret_cast<uintptr_t>(at.devicePointer) & 15) ? nullptr : at.devicePointer;
}

bool is_host_ptr(const void* p) {
    if (!p) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return true;
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

struct LayerState {
    int len = 0;
    int pending_min_page = INT_MAX;  // lowest page written to the host since the copy stream last waited
    bool hist_recorded = false;
};

enum TimedKind { kTDecodeRes, kTDecodeRing, kTMerge, kTAppend, kTChunkMma, kTDecodeZc, kTChunkZc };

struct Timed {
    cudaEvent_t a, b;
    int kind;
    uint64_t bytes;
};

}  // namespace

void kvs::set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

struct kvs_s {
    kvs_config cfg{};
    int device = 0;
    size_t page_bytes = 0;
    long P_max = 0;
    size_t host_bytes = 0;
    uint8_t* host = nullptr;
    uint8_t* host_dev = nullptr;
    uint8_t* arena = nullptr;
    ArenaLayout lay{};
    uint8_t* resident = nullptr;
    uint8_t* ring = nullptr;
    PartialBuffers part{};
    __half *stage_q = nullptr, *stage_k = nullptr, *stage_v = nullptr;
    float *stage_out = nullptr, *stage_lse = nullptr;
    int* err_word = nullptr;
    CUtensorMap map_res{}, map_ring{}, map_aux{};
    // phase arena: the phase, its width (widest batch), the allocation, the
    // auxiliary layers' pinned pages (at the top) and the kvs_pin bytes below
    bool phase_arena = false;
    int phase = KVS_PHASE_PREFILL;
    int width = 1;
    int aux_R = 0;                   // auxiliary layers' resident pages (configured)
    bool draft_active = true;
    size_t alloc_bytes = 0;
    size_t pin_bytes = 0;
    uint8_t* aux = nullptr;          // auxiliary layers' resident region
    void* encode_fn = nullptr;       // cuTensorMapEncodeTiled
    cudaStream_t cs = nullptr;       // copy stream (H2D ring)
    cudaStream_t rs = nullptr;       // side stream: resident-page attention (lowest priority)
    cudaStream_t xs = nullptr;       // ring attention stream (highest priority)
    cudaStream_t zs = nullptr;       // in-place (zero-copy) attention of streamed pages (lowest)
    cudaEvent_t ev_fork = nullptr, ev_res = nullptr, ev_ring = nullptr, ev_zc = nullptr, ev_join = nullptr;
    size_t partial_capacity = 0;     // (split x row) records
    int n_groups = 0;
    std::vector<cudaEvent_t> ev_full, ev_free, ev_hist;
    std::vector<char> free_valid;
    // stream-capture bookkeeping: the capture id (0 = none) in which each
    // ring-free / history event was last recorded, the capture the copy stream
    // has joined, and whether a capture happened since the last plain call
    std::vector<unsigned long long> free_cap, hist_cap;
    unsigned long long cs_cap = 0;
    bool capture_seen = false;
    uint64_t ring_ctr = 0;
    std::vector<RingCopy> ring_plan;  // the current call's ring schedule
    std::vector<LayerState> layers;
    kvs_stats stats{};
    std::vector<Timed> timed;
    std::vector<cudaEvent_t> ev_pool;
    std::string err;
};

namespace {

int fail(kvs_t* kv, int code, const std::string& why) {
    if (kv) kv->err = why;
    g_last_error = why;
    return code;
}

#define KVS_CK(kv, call)                                                                    \
    do {                                                                                    \
        cudaError_t e_ = (call);                                                            \
        if (e_ != cudaSuccess)                                                              \
            return fail((kv), KVS_E_CUDA, fmt("%s failed: %s", #call, cudaGetErrorString(e_))); \
    } while (0)

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

cudaEvent_t pool_event(kvs_t* kv) {
    if (!kv->ev_pool.empty()) {
        cudaEvent_t e = kv->ev_pool.back();
        kv->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// id of the capture `s` is recording into, 0 when it is not capturing
unsigned long long capture_id(cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    unsigned long long id = 0;
    if (cudaStreamGetCaptureInfo(s, &st, &id) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return st == cudaStreamCaptureStatusActive ? id : 0;
}

bool profiling(const kvs_t* kv, cudaStream_t s) {
    if (!(kv->cfg.flags & KVS_FLAG_PROFILE)) return false;
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &st);
    return st == cudaStreamCaptureStatusNone;
}

struct TimedScope {
    kvs_t* kv;
    cudaStream_t s;
    bool on;
    Timed t{};
    TimedScope(kvs_t* k, cudaStream_t st, int kind, uint64_t bytes) : kv(k), s(st) {
        on = profiling(k, st);
        if (on) {
            t.a = pool_event(k);
            t.b = pool_event(k);
            t.kind = kind;
            t.bytes = bytes;
            cudaEventRecord(t.a, s);
        }
    }
    ~TimedScope();
};

void fold_timed_upto(kvs_t* kv, size_t n);

// fold the leading records whose end event has completed (non-blocking)
void fold_completed(kvs_t* kv) {
    size_t n = 0;
    while (n < kv->timed.size() && cudaEventQuery(kv->timed[n].b) == cudaSuccess) ++n;
    cudaGetLastError();
    fold_timed_upto(kv, n);
}

TimedScope::~TimedScope() {
    if (on) {
        cudaEventRecord(t.b, s);
        kv->timed.push_back(t);
        if (kv->timed.size() >= 2048) fold_completed(kv);
    }
}

int encode_map(kvs_t* kv, EncodeTiledFn fn, CUtensorMap* map, void* base, uint64_t rows) {
    if (rows == 0) return KVS_OK;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(kv, KVS_E_CUDA, fmt("cuTensorMapEncodeTiled failed (%d)", (int)r));
    return KVS_OK;
}

// The arena laid out for resident count R and the phase width: pointers into
// the allocation, tensor maps, partial capacity.  The auxiliary layers' pages
// sit at the top of the allocation while the draft is active.
int apply_layout(kvs_t* kv, long R, int width) {
    kvs_config c = kv->cfg;
    c.n_resident_pages = (int)R;
    c.max_q_tokens = width;
    const ArenaLayout L = arena_layout(c);
    kv->lay = L;
    kv->cfg.n_resident_pages = (int)R;
    kv->width = width;
    kv->resident = kv->arena + L.resident;
    kv->ring = kv->arena + L.ring;
    kv->part.ml = reinterpret_cast<float2*>(kv->arena + L.part_ml);
    kv->part.acc = reinterpret_cast<float*>(kv->arena + L.part_acc);
    kv->stage_q = reinterpret_cast<__half*>(kv->arena + L.stage_q);
    kv->stage_k = reinterpret_cast<__half*>(kv->arena + L.stage_kv);
    kv->stage_v = kv->stage_k + (size_t)width * c.n_kv_heads * kHeadDim;
    kv->stage_out = reinterpret_cast<float*>(kv->arena + L.stage_out);
    kv->stage_lse = reinterpret_cast<float*>(kv->arena + L.stage_lse);
    kv->err_word = reinterpret_cast<int*>(kv->arena + L.err);
    kv->partial_capacity = partial_records(c);
    auto enc = reinterpret_cast<EncodeTiledFn>(kv->encode_fn);
    const uint64_t head_rows = (uint64_t)page_head_bytes(c.type_v, c.type_k) / 128;
    const uint64_t res_rows = (uint64_t)target_layers(c) * R * c.n_kv_heads * head_rows;
    const uint64_t ring_rows = (uint64_t)c.n_ring_slots * c.n_kv_heads * head_rows;
    if (encode_map(kv, enc, &kv->map_res, kv->resident, res_rows) != KVS_OK) return KVS_E_CUDA;
    if (encode_map(kv, enc, &kv->map_ring, kv->ring, ring_rows) != KVS_OK) return KVS_E_CUDA;
    kv->aux = nullptr;
    if (c.n_aux_layers > 0 && kv->draft_active) {
        kv->aux = kv->arena + kv->alloc_bytes - aux_region_bytes(c);
        const uint64_t aux_rows = (uint64_t)c.n_aux_layers * c.aux_resident_pages * c.n_kv_heads * head_rows;
        if (encode_map(kv, enc, &kv->map_aux, kv->aux, aux_rows) != KVS_OK) return KVS_E_CUDA;
    }
    return KVS_OK;
}

// where a layer's resident pages live: region base, slots per layer, global
// slot index of the layer's slot 0 in the region's tensor map, the map
struct LayerRes {
    uint8_t* base;
    long R;
    long slot_base;
    const CUtensorMap* map;
};
LayerRes layer_res(kvs_t* kv, int layer) {
    const int LT = target_layers(kv->cfg);
    if (layer < LT) {
        const long R = kv->cfg.n_resident_pages;
        return {kv->resident + (size_t)layer * R * kv->page_bytes, R, (long)layer * R, &kv->map_res};
    }
    const long R = kv->cfg.aux_resident_pages;
    const int a = layer - LT;
    return {kv->aux + (size_t)a * R * kv->page_bytes, R, (long)a * R, &kv->map_aux};
}
bool aux_layer(const kvs_t* kv, int layer) { return layer >= target_layers(kv->cfg); }

// copy a layer's resident pages (the newest R of its history) from the
// authoritative host history into their slots (page p -> slot p mod R), one
// copy per run of consecutive slots
int recopy_layer(kvs_t* kv, int layer, cudaStream_t s) {
    const LayerRes r = layer_res(kv, layer);
    const long P = pages_for(kv->layers[layer].len);
    long p = std::max(0L, P - r.R);
    while (p < P) {
        long q = p + 1;
        while (q < P && (q % r.R) != 0) ++q;  // slots p mod R .. stay consecutive until the wrap
        const size_t src = ((size_t)layer * kv->P_max + (size_t)p) * kv->page_bytes;
        const cudaError_t e = cudaMemcpyAsync(r.base + (size_t)(p % r.R) * kv->page_bytes, kv->host + src,
                                              (size_t)(q - p) * kv->page_bytes, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return fail(kv, KVS_E_CUDA, fmt("cudaMemcpyAsync: %s", cudaGetErrorString(e)));
        p = q;
    }
    return KVS_OK;
}

// status of a phase arena laid out for resident count R and `width`
void fill_status(const kvs_config& c, long R, int width, size_t alloc, size_t pin, bool draft, int phase,
                 kvs_arena_status* st) {
    kvs_config cw = c;
    cw.n_resident_pages = (int)R;
    cw.max_q_tokens = width;
    const ArenaLayout L = arena_layout(cw);
    std::memset(st, 0, sizeof(*st));
    st->phase = phase;
    st->width = width;
    st->n_resident_pages = (int)R;
    st->draft_active = draft ? 1 : 0;
    st->aux_resident_pages = draft ? c.aux_resident_pages : 0;
    st->phase_arena = (c.flags & KVS_FLAG_PHASE_ARENA) ? 1 : 0;
    st->arena_bytes = alloc;
    st->resident_bytes = L.ring - L.resident;
    st->ring_bytes = L.part_ml - L.ring;
    st->compute_bytes = L.total - L.part_ml;
    st->aux_bytes = draft ? aux_region_bytes(c) : 0;
    st->pinned_bytes = pin;
    const size_t used = L.total + st->aux_bytes + pin;
    st->free_bytes = alloc > used ? alloc - used : 0;
}

void release(kvs_t* kv) {
    if (!kv) return;
    DeviceGuard g(kv->device);
    for (auto& t : kv->timed) { cudaEventDestroy(t.a); cudaEventDestroy(t.b); }
    for (auto e : kv->ev_pool) cudaEventDestroy(e);
    for (auto e : kv->ev_full) if (e) cudaEventDestroy(e);
    for (auto e : kv->ev_free) if (e) cudaEventDestroy(e);
    for (auto e : kv->ev_hist) if (e) cudaEventDestroy(e);
    if (kv->ev_fork) cudaEventDestroy(kv->ev_fork);
    if (kv->ev_res) cudaEventDestroy(kv->ev_res);
    if (kv->ev_ring) cudaEventDestroy(kv->ev_ring);
    if (kv->ev_zc) cudaEventDestroy(kv->ev_zc);
    if (kv->ev_join) cudaEventDestroy(kv->ev_join);
    if (kv->zs) cudaStreamDestroy(kv->zs);
    if (kv->xs) cudaStreamDestroy(kv->xs);
    if (kv->cs) cudaStreamDestroy(kv->cs);
    if (kv->rs) cudaStreamDestroy(kv->rs);
    if (kv->arena) cudaFree(kv->arena);
    if (kv->host) cudaFreeHost(kv->host);
    delete kv;
}

// bounded host wait on an event
int wait_event(kvs_t* kv, cudaEvent_t e, double timeout_s) {
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        cudaError_t q = cudaEventQuery(e);
        if (q == cudaSuccess) return KVS_OK;
        if (q != cudaErrorNotReady) return fail(kv, KVS_E_CUDA, fmt("cudaEventQuery: %s", cudaGetErrorString(q)));
        const double el = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
        if (el > timeout_s) return fail(kv, KVS_E_TIMEOUT, "bounded wait for GPU work timed out");
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
}

int sync_all(kvs_t* kv, cudaStream_t user, double timeout_s) {
    int rc = KVS_OK;
    for (cudaStream_t st : {kv->cs, user, kv->rs, kv->xs, kv->zs}) {
        cudaEvent_t e = pool_event(kv);
        KVS_CK(kv, cudaEventRecord(e, st));
        if (rc == KVS_OK) rc = wait_event(kv, e, timeout_s);
        kv->ev_pool.push_back(e);
    }
    if (rc != KVS_OK) return rc;
    int err = 0;
    KVS_CK(kv, cudaMemcpy(&err, kv->err_word, sizeof(int), cudaMemcpyDeviceToHost));
    if (err) return fail(kv, KVS_E_TIMEOUT, fmt("a kernel's bounded wait gave up (error word %d)", err));
    return KVS_OK;
}

void fold_timed_upto(kvs_t* kv, size_t n) {
    for (size_t i = 0; i < n; ++i) {
        Timed& t = kv->timed[i];
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, t.a, t.b) != cudaSuccess) { cudaGetLastError(); ms = 0.f; }
        switch (t.kind) {
            case kTDecodeRes: kv->stats.ms_decode_resident += ms; kv->stats.n_decode_resident++;
                              kv->stats.bytes_decode_resident += t.bytes; break;
            case kTDecodeRing: kv->stats.ms_decode_ring += ms; kv->stats.n_decode_ring++;
                               kv->stats.bytes_decode_ring += t.bytes; break;
            case kTMerge: kv->stats.ms_merge += ms; kv->stats.n_merge++; break;
            case kTAppend: kv->stats.ms_append += ms; kv->stats.n_append++; break;
            case kTChunkMma: kv->stats.ms_chunk_mma += ms; kv->stats.n_chunk_mma++; break;
            case kTDecodeZc: kv->stats.ms_decode_zc += ms; kv->stats.n_decode_zc++;
                             kv->stats.bytes_decode_zc += t.bytes; break;
            case kTChunkZc: kv->stats.ms_chunk_zc += ms; kv->stats.n_chunk_zc++;
                            kv->stats.bytes_chunk_zc += t.bytes; break;
        }
        kv->ev_pool.push_back(t.a);
        kv->ev_pool.push_back(t.b);
    }
    kv->timed.erase(kv->timed.begin(), kv->timed.begin() + n);
}

void fold_timed(kvs_t* kv) { fold_timed_upto(kv, kv->timed.size()); }

// Re-lend a phase arena: the phase width, the kvs_pin bytes and the draft's
// state decide the layout.  Fits the target's resident count first (the state
// is untouched if nothing fits), waits for the handle's work, lays the arena
// out and copies from the host history every page that is resident in the new
// layout but was not (all target pages when R changes; the auxiliary layers'
// pages when the draft comes back).
int relayout(kvs_t* kv, int width, size_t pin_bytes, bool draft_active, cudaStream_t s) {
    if (capture_id(s)) return fail(kv, KVS_E_INVAL, "the arena cannot be re-lent during stream capture");
    kvs_config c = kv->cfg;
    c.max_q_tokens = width;
    const size_t aux_bytes = (draft_active && c.n_aux_layers > 0) ? aux_region_bytes(c) : 0;
    if (aux_bytes + pin_bytes >= kv->alloc_bytes)
        return fail(kv, KVS_E_ARENA, "the pinned region would fill the arena");
    const long R = resident_fit(c, kv->alloc_bytes - aux_bytes - pin_bytes, kv->P_max);
    if (R < 1)
        return fail(kv, KVS_E_ARENA, fmt("no resident page fits a width-%d phase beside %zu pinned bytes", width,
                                         aux_bytes + pin_bytes));
    int rc = sync_all(kv, s, 60.0);
    if (rc != KVS_OK) return rc;
    const bool r_changed = R != kv->cfg.n_resident_pages;
    const bool aux_back = draft_active && !kv->draft_active;
    kv->pin_bytes = pin_bytes;
    kv->draft_active = draft_active;
    if (r_changed || width != kv->width || aux_back || !draft_active) {
        if (apply_layout(kv, R, width) != KVS_OK) return KVS_E_CUDA;
        KVS_CK(kv, cudaMemsetAsync(kv->err_word, 0, sizeof(int), s));
    }
    const int LT = target_layers(kv->cfg);
    if (r_changed)
        for (int l = 0; l < LT; ++l)
            if ((rc = recopy_layer(kv, l, s)) != KVS_OK) return rc;
    if (aux_back)
        for (int l = LT; l < kv->cfg.n_layers; ++l)
            if ((rc = recopy_layer(kv, l, s)) != KVS_OK) return rc;
    return KVS_OK;
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

int kvs_resolve_config(const kvs_config* in, kvs_config* out, size_t* host_bytes) {
    std::string why;
    int rc = resolve(in, out, host_bytes, why);
    if (rc != KVS_OK) g_last_error = why;
    return rc;
}

size_t kvs_page_bytes(const kvs_config* cfg) {
    return cfg ? (size_t)cfg->n_kv_heads * page_head_bytes(cfg->type_v, cfg->type_k) : 0;
}

int kvs_plan_page(const kvs_config* c, int n_tokens, int page, int* kind, int* index) {
    if (!c || !kind || !index || n_tokens < 0 || c->n_resident_pages < 1) {
        g_last_error = "kvs_plan_page: bad arguments (config must be resolved)";
        return KVS_E_INVAL;
    }
    return plan_page(*c, n_tokens, page, kind, index);
}

int kvs_plan_ring(const kvs_config* c, int n_q, int s_ring, long long ring_ctr0, int* page0, int* pages,
                  int* slot0, int max_copies) {
    if (!c || n_q < 1 || s_ring < 0 || ring_ctr0 < 0 || max_copies < 0 ||
        (max_copies > 0 && (!page0 || !pages || !slot0)) || c->n_ring_slots < 0 || c->chunk_pages < 0 ||
        (c->n_ring_slots > 0 && c->chunk_pages < 1)) {
        g_last_error = "kvs_plan_ring: bad arguments (config must be resolved)";
        return KVS_E_INVAL;
    }
    std::vector<RingCopy> plan;
    plan_ring(*c, n_q, s_ring, ring_ctr0, plan);
    for (int i = 0; i < (int)plan.size() && i < max_copies; ++i) {
        page0[i] = (int)plan[i].page0;
        pages[i] = plan[i].pages;
        slot0[i] = plan[i].slot0;
    }
    return (int)plan.size();
}

int kvs_eject_init(kvs_eject_params* p, kvs_eject_state* s) {
    if (!p || !s || p->keep_pages < 0 || p->reenable_pages < 0 || p->stable_decodes < 0 ||
        p->capacity_pages < 0) {
        g_last_error = "kvs_eject_init: null pointer or negative field";
        return KVS_E_INVAL;
    }
    if (p->reenable_pages == 0) p->reenable_pages = 8;
    if (p->stable_decodes == 0) p->stable_decodes = 4;
    if (p->keep_pages == 0 && p->capacity_pages == 0) {
        g_last_error = "kvs_eject_init: the threshold (keep_pages, else capacity_pages) is zero";
        return KVS_E_INVAL;
    }
    s->draft_active = 1;
    s->streak = 0;
    return KVS_OK;
}

int kvs_eject_step(const kvs_eject_params* p, kvs_eject_state* s, int working_pages) {
    if (!p || !s || working_pages < 0 || p->stable_decodes < 1 || p->reenable_pages < 0) {
        g_last_error = "kvs_eject_step: bad arguments (call kvs_eject_init first)";
        return KVS_E_INVAL;
    }
    const long threshold = p->keep_pages > 0 ? p->keep_pages : p->capacity_pages;
    const bool cond = s->draft_active ? (working_pages > threshold)
                                      : ((long)working_pages <= threshold - p->reenable_pages);
    s->streak = cond ? s->streak + 1 : 0;
    if (s->streak < p->stable_decodes) return 0;
    s->draft_active = !s->draft_active;
    s->streak = 0;
    return 1;
}

int kvs_draft_capacity_pages(const kvs_config* cfg, size_t pinned_bytes, int* pages) {
    if (!cfg || !pages) { g_last_error = "kvs_draft_capacity_pages: null argument"; return KVS_E_INVAL; }
    if (cfg->arena_bytes == 0) {
        g_last_error = "kvs_draft_capacity_pages: needs a fixed arena_bytes";
        return KVS_E_INVAL;
    }
    if (pinned_bytes >= cfg->arena_bytes) {
        g_last_error = "kvs_draft_capacity_pages: the pinned reservation fills the arena";
        return KVS_E_ARENA;
    }
    kvs_config c = *cfg;
    c.n_resident_pages = 0;
    c.arena_bytes -= pinned_bytes;
    kvs_config r;
    std::string why;
    const int rc = resolve(&c, &r, nullptr, why);
    if (rc != KVS_OK) { g_last_error = why; return rc; }
    *pages = r.n_resident_pages;
    return KVS_OK;
}

int kvs_create(const kvs_config* cfg, int device, kvs_t** out) {
    if (!out) return fail(nullptr, KVS_E_INVAL, "kvs_create: null out");
    *out = nullptr;
    kvs_config c;
    size_t host_bytes = 0;
    std::string why;
    int rc = resolve(cfg, &c, &host_bytes, why);
    if (rc != KVS_OK) return fail(nullptr, rc, why);
    int n_dev = 0;
    if (cudaGetDeviceCount(&n_dev) != cudaSuccess || n_dev == 0) {
        cudaGetLastError();
        return fail(nullptr, KVS_E_CUDA, "no CUDA device: libkvs has no CPU fallback");
    }
    if (device < 0 || device >= n_dev) return fail(nullptr, KVS_E_INVAL, fmt("device %d out of range", device));
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess || prop.major < 10)
        return fail(nullptr, KVS_E_INVAL, "libkvs is built for sm_100a (B200)");

    kvs_t* kv = new kvs_t();
    kv->cfg = c;
    kv->device = device;
    kv->page_bytes = (size_t)c.n_kv_heads * page_head_bytes(c.type_v, c.type_k);
    kv->P_max = pages_for(c.max_ctx);
    kv->host_bytes = host_bytes;
    kv->lay = arena_layout(c);
    // a phase arena allocates its whole budget and starts in the prefill phase
    // (the widest batch); otherwise the arena is the exact fit
    kv->phase_arena = (c.flags & KVS_FLAG_PHASE_ARENA) != 0;
    kv->alloc_bytes = kv->phase_arena ? c.arena_bytes : kv->lay.total;
    kv->phase = KVS_PHASE_PREFILL;
    kv->width = c.max_q_tokens;
    DeviceGuard g(device);
    auto bail = [&](int code, const std::string& w) {
        g_last_error = w;
        release(kv);
        return code;
    };
    cudaError_t e = cudaHostAlloc(reinterpret_cast<void**>(&kv->host), host_bytes,
                                  cudaHostAllocMapped | cudaHostAllocPortable);
    if (e != cudaSuccess) {
        kv->host = nullptr;
        return bail(KVS_E_NOMEM, fmt("cudaHostAlloc(%zu B pinned history) failed: %s", host_bytes, cudaGetErrorString(e)));
    }
    std::memset(kv->host, 0, host_bytes);
    e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&kv->host_dev), kv->host, 0);
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("cudaHostGetDevicePointer: %s", cudaGetErrorString(e)));
    e = cudaMalloc(reinterpret_cast<void**>(&kv->arena), kv->alloc_bytes);
    if (e != cudaSuccess) {
        kv->arena = nullptr;
        return bail(KVS_E_ARENA, fmt("cudaMalloc(arena %zu B) failed: %s", kv->alloc_bytes, cudaGetErrorString(e)));
    }
    e = cudaMemset(kv->arena, 0, kv->alloc_bytes);
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("cudaMemset: %s", cudaGetErrorString(e)));

    e = cudaStreamCreateWithFlags(&kv->cs, cudaStreamNonBlocking);
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("cudaStreamCreate: %s", cudaGetErrorString(e)));
    // the ring's attention kernels free ring slots for the copy engine, so they
    // run at the highest priority; resident-page attention fills in behind them
    int prio_low = 0, prio_high = 0;
    cudaDeviceGetStreamPriorityRange(&prio_low, &prio_high);
    e = cudaStreamCreateWithPriority(&kv->rs, cudaStreamNonBlocking, prio_low);
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("cudaStreamCreate: %s", cudaGetErrorString(e)));
    e = cudaStreamCreateWithPriority(&kv->xs, cudaStreamNonBlocking, prio_high);
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("cudaStreamCreate: %s", cudaGetErrorString(e)));
    e = cudaStreamCreateWithPriority(&kv->zs, cudaStreamNonBlocking, prio_low);
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("cudaStreamCreate: %s", cudaGetErrorString(e)));
    if (cudaEventCreateWithFlags(&kv->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&kv->ev_res, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&kv->ev_ring, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&kv->ev_zc, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&kv->ev_join, cudaEventDisableTiming) != cudaSuccess)
        return bail(KVS_E_CUDA, "cudaEventCreate failed");
    kv->n_groups = c.n_ring_slots > 0 ? c.n_ring_slots / c.chunk_pages : 0;
    kv->ev_full.assign(kv->n_groups, nullptr);
    kv->ev_free.assign(kv->n_groups, nullptr);
    kv->free_valid.assign(kv->n_groups, 0);
    kv->free_cap.assign(kv->n_groups, 0);
    for (int i = 0; i < kv->n_groups; ++i) {
        if (cudaEventCreateWithFlags(&kv->ev_full[i], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&kv->ev_free[i], cudaEventDisableTiming) != cudaSuccess)
            return bail(KVS_E_CUDA, "cudaEventCreate failed");
    }
    kv->ev_hist.assign(c.n_layers, nullptr);
    for (int i = 0; i < c.n_layers; ++i)
        if (cudaEventCreateWithFlags(&kv->ev_hist[i], cudaEventDisableTiming) != cudaSuccess)
            return bail(KVS_E_CUDA, "cudaEventCreate failed");
    kv->layers.assign(c.n_layers, LayerState{});
    kv->hist_cap.assign(c.n_layers, 0);

    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr);
    if (e != cudaSuccess || qr != cudaDriverEntryPointSuccess || !fn)
        return bail(KVS_E_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    kv->encode_fn = fn;
    if (apply_layout(kv, c.n_resident_pages, c.max_q_tokens) != KVS_OK) return bail(KVS_E_CUDA, kv->err);
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return bail(KVS_E_CUDA, fmt("create sync: %s", cudaGetErrorString(e)));
    if (getenv("KVS_LOG")) {
        fprintf(stderr,
                "kvs: pool created: %d layer(s), %d resident pages/layer, %d ring slots (chunk %d), "
                "page %zu B, arena %.2f MiB%s, pinned history %.2f MiB, device %d\n",
                c.n_layers, c.n_resident_pages, c.n_ring_slots, c.chunk_pages, kv->page_bytes,
                kv->alloc_bytes / 1048576.0, kv->phase_arena ? " (phase arena)" : "", host_bytes / 1048576.0,
                device);
    }
    *out = kv;
    return KVS_OK;
}

void kvs_destroy(kvs_t* kv) {
    if (!kv) return;
    {
        DeviceGuard g(kv->device);
        for (cudaStream_t st : {kv->cs, kv->rs, kv->xs, kv->zs}) {
            cudaEvent_t e = pool_event(kv);
            if (e && st && cudaEventRecord(e, st) == cudaSuccess) wait_event(kv, e, 60.0);
            if (e) kv->ev_pool.push_back(e);
        }
        cudaDeviceSynchronize();
    }
    release(kv);
}

int kvs_append(kvs_t* kv, int layer, int pos0, int n_tok, const void* k_f16, const void* v_f16,
               void* stream) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    const kvs_config& c = kv->cfg;
    if (layer < 0 || layer >= c.n_layers) return fail(kv, KVS_E_INVAL, fmt("layer %d out of range", layer));
    if (n_tok < 1) return fail(kv, KVS_E_INVAL, "n_tok must be >= 1");
    if (!k_f16 || !v_f16) return fail(kv, KVS_E_INVAL, "null K/V");
    if (aux_layer(kv, layer) && !kv->draft_active)
        return fail(kv, KVS_E_INVAL, "auxiliary layers are ejected (kvs_draft_restore brings them back)");
    const bool host_k = is_host_ptr(k_f16), host_v = is_host_ptr(v_f16);
    // host K/V go through staging buffers sized for the phase's width; device
    // K/V may be any width (history pre-fill)
    if ((host_k || host_v) && n_tok > kv->width)
        return fail(kv, KVS_E_WIDTH, fmt("append batch too wide: %d > width %d", n_tok, kv->width));
    LayerState& ls = kv->layers[layer];
    if (pos0 < 0 || pos0 > ls.len)
        return fail(kv, KVS_E_ORDER, fmt("append at %d is not contiguous with length %d", pos0, ls.len));
    if ((long)pos0 + n_tok > c.max_ctx)
        return fail(kv, KVS_E_INVAL, fmt("append beyond max_ctx (%d)", c.max_ctx));
    DeviceGuard g(kv->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Stream capture: the copy stream joins the capture here, ahead of the
    // append kernel, so a captured step's first ring copy starts with the
    // graph instead of after the append.  The copies read only history pages
    // that no append of this capture has written (kvs_attend waits for the
    // append's history write when one of its pages is streamed).
    {
        const unsigned long long cap = capture_id(s);
        if (cap && c.n_ring_slots > 0 && kv->cs_cap != cap) {
            KVS_CK(kv, cudaEventRecord(kv->ev_fork, s));
            KVS_CK(kv, cudaStreamWaitEvent(kv->cs, kv->ev_fork, 0));
            // joined straight back, so a capture that ends before any attend
            // call leaves no stream behind (the caller's stream gains no wait:
            // the copy stream holds nothing yet)
            KVS_CK(kv, cudaEventRecord(kv->ev_join, kv->cs));
            KVS_CK(kv, cudaStreamWaitEvent(s, kv->ev_join, 0));
            kv->cs_cap = cap;
            kv->capture_seen = true;
        }
    }
    const size_t kv_elems = (size_t)n_tok * c.n_kv_heads * kHeadDim;
    const __half* k = static_cast<const __half*>(k_f16);
    const __half* v = static_cast<const __half*>(v_f16);
    // pinned host K/V: the append kernel reads them in place over PCIe;
    // pageable ones are staged by the copy engine
    if (host_k) {
        const void* a = pinned_alias16(k_f16);
        if (a) {
            k = static_cast<const __half*>(a);
        } else {
            KVS_CK(kv, cudaMemcpyAsync(kv->stage_k, k_f16, kv_elems * 2, cudaMemcpyHostToDevice, s));
            k = kv->stage_k;
        }
    }
    if (host_v) {
        const void* a = pinned_alias16(v_f16);
        if (a) {
            v = static_cast<const __half*>(a);
        } else {
            KVS_CK(kv, cudaMemcpyAsync(kv->stage_v, v_f16, kv_elems * 2, cudaMemcpyHostToDevice, s));
            v = kv->stage_v;
        }
    }
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 7)
        return fail(kv, KVS_E_INVAL, "K/V must be 8-byte aligned");

    const LayerRes lr = layer_res(kv, layer);
    const long R = lr.R;
    const long P_old = pages_for(ls.len), P_new = pages_for((long)pos0 + n_tok);
    const long f_old = std::max(0L, P_old - R), f_new = std::max(0L, P_new - R);
    // pages that re-enter the resident set after a roll-back and keep tokens
    // below pos0 are copied back from the authoritative host history
    for (long p = f_new; p < P_new; ++p) {
        const bool was_res = (p >= f_old && p < P_old);
        if (!was_res && p * kPageTokens < pos0) {
            const size_t src = ((size_t)layer * kv->P_max + p) * kv->page_bytes;
            uint8_t* dst = lr.base + (size_t)(p % R) * kv->page_bytes;
            KVS_CK(kv, cudaMemcpyAsync(dst, kv->host + src, kv->page_bytes, cudaMemcpyHostToDevice, s));
        }
    }
    AppendArgs a;
    a.k = k;
    a.v = v;
    a.host_layer = kv->host_dev + (size_t)layer * kv->P_max * kv->page_bytes;
    a.res_layer = lr.base;
    a.n_tok = n_tok;
    a.pos0 = pos0;
    a.n_kv = c.n_kv_heads;
    a.n_resident = (int)R;
    a.first_resident_page = (int)f_new;
    a.page_bytes = kv->page_bytes;
    a.v_type = c.type_v;
    a.k_type = c.type_k;
    {
        TimedScope ts(kv, s, kTAppend, 0);
        KVS_CK(kv, launch_append(a, s));
    }
    kv->stats.kernel_launches++;
    KVS_CK(kv, cudaEventRecord(kv->ev_hist[layer], s));
    kv->hist_cap[layer] = capture_id(s);
    if (kv->hist_cap[layer]) kv->capture_seen = true;
    ls.hist_recorded = true;
    ls.pending_min_page = std::min(ls.pending_min_page, pos0 / kPageTokens);
    ls.len = pos0 + n_tok;
    kv->stats.appends++;
    kv->stats.tokens_appended += n_tok;
    return KVS_OK;
}

int kvs_attend(kvs_t* kv, int layer, int pos0, int n_q, const void* q_f16, float* out, float* lse,
               void* stream) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    const kvs_config& c = kv->cfg;
    if (layer < 0 || layer >= c.n_layers) return fail(kv, KVS_E_INVAL, fmt("layer %d out of range", layer));
    if (n_q < 1) return fail(kv, KVS_E_INVAL, "n_q must be >= 1");
    if (n_q > kv->width)
        return fail(kv, KVS_E_WIDTH, kv->phase_arena && kv->phase == KVS_PHASE_DECODE
                                         ? fmt("phase arena decode batch too wide: %d > width %d", n_q, kv->width)
                                         : fmt("decode batch too wide: %d > max_q_tokens %d", n_q, kv->width));
    if (!q_f16 || !out) return fail(kv, KVS_E_INVAL, "null q/out");
    if (aux_layer(kv, layer) && !kv->draft_active)
        return fail(kv, KVS_E_INVAL, "auxiliary layers are ejected (kvs_draft_restore brings them back)");
    LayerState& ls = kv->layers[layer];
    if (pos0 < 0 || (long)pos0 + n_q > ls.len)
        return fail(kv, KVS_E_ORDER, fmt("queries %d..%d beyond the history (length %d)", pos0, pos0 + n_q - 1, ls.len));
    DeviceGuard g(kv->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int rows = n_q * c.n_q_heads;
    const bool tc = use_tcgen05(c, n_q);
    // Device buffers go to the kernels as they are, so their addresses must
    // suit the kernels' vector accesses: Q is read in 8-byte words by the
    // decode kernel and 16-byte words by the tensor-core kernel; out is
    // written in 16-byte words when the many-row merge runs (>= 1024 rows).
    // Host buffers are staged or aliased only when 16-byte aligned.
    {
        const uintptr_t qa = reinterpret_cast<uintptr_t>(q_f16), oa = reinterpret_cast<uintptr_t>(out);
        if (!is_host_ptr(q_f16) && (qa & (tc ? 15 : 7)))
            return fail(kv, KVS_E_INVAL, tc ? "q must be 16-byte aligned for multi-token attention"
                                            : "q must be 8-byte aligned");
        if (!is_host_ptr(out) && (oa & (rows >= kMergeRowsMin ? 15 : 3)))
            return fail(kv, KVS_E_INVAL, rows >= kMergeRowsMin ? "out must be 16-byte aligned for >= 1024 query rows"
                                                               : "out must be 4-byte aligned");
        if (lse && !is_host_ptr(lse) && (reinterpret_cast<uintptr_t>(lse) & 3))
            return fail(kv, KVS_E_INVAL, "lse must be 4-byte aligned");
    }
    const __half* q = static_cast<const __half*>(q_f16);
    if (is_host_ptr(q_f16)) {
        // pinned: one small copy kernel pulls Q over PCIe; pageable: copy engine
        const void* a = pinned_alias16(q_f16);
        if (a) KVS_CK(kv, launch_copy16(kv->stage_q, a, (size_t)rows * kHeadDim * 2, s));
        else KVS_CK(kv, cudaMemcpyAsync(kv->stage_q, q_f16, (size_t)rows * kHeadDim * 2, cudaMemcpyHostToDevice, s));
        q = kv->stage_q;
    }
    // pinned host out/lse: the merge kernel writes them in place over PCIe
    float* out_alias = is_host_ptr(out) ? static_cast<float*>(const_cast<void*>(pinned_alias16(out))) : nullptr;
    float* lse_alias = (lse && is_host_ptr(lse)) ? static_cast<float*>(const_cast<void*>(pinned_alias16(lse))) : nullptr;
    const bool host_out = is_host_ptr(out) && !out_alias;
    const bool host_lse = lse && is_host_ptr(lse) && !lse_alias;
    float* dout = out_alias ? out_alias : (host_out ? kv->stage_out : out);
    float* dlse = lse ? (lse_alias ? lse_alias : (host_lse ? kv->stage_lse : lse)) : nullptr;

    const LayerRes lres = layer_res(kv, layer);
    const long R = lres.R;
    const long P = pages_for(ls.len);
    const long R_eff = std::min(R, P);
    const long first_res = P - R_eff;
    const long S = first_res;
    const long S_zc = zero_copy_pages(c, n_q, S);  // streamed pages read in place
    const long S_ring = S - S_zc;                  // streamed pages copied through the ring

    DecodeArgs d{};
    d.v_type = c.type_v;
    d.k_type = c.type_k;
    d.len = ls.len;
    d.pos0 = pos0;
    d.n_q = n_q;
    d.q = q;
    d.q_scale = (float)(1.4426950408889634 / std::sqrt((double)kHeadDim));
    d.n_qh = c.n_q_heads;
    d.n_kv = c.n_kv_heads;
    d.group = c.n_q_heads / c.n_kv_heads;
    d.part = kv->part;
    d.n_rows = rows;
    d.err = kv->err_word;

    // split counts first: the partial buffer must hold every (split, row) record
    if ((size_t)count_splits(c, n_q, R_eff, S) * rows > kv->partial_capacity ||
        (size_t)rows > (size_t)kv->width * c.n_q_heads)
        return fail(kv, KVS_E_INVAL, "internal: partial buffer too small for this call");
    // With profiling on, every kernel runs on the caller's stream so that the
    // events around a launch time that launch alone.
    const bool prof = profiling(kv, s);
    const unsigned long long cap = capture_id(s);
    cudaStream_t rstream = prof ? s : kv->rs;
    cudaStream_t xstream = prof ? s : kv->xs;
    cudaStream_t zstream = prof ? s : kv->zs;
    // 1) resident pages, attended in place on the side stream so they overlap
    //    the ring pipeline below
    int split_base = 0;
    {
        d.region = lres.base;
        d.region_slot_base = (int)lres.slot_base;
        d.region_slots = (int)R;
        d.slot0 = (int)(first_res % R);
        d.page0 = (int)first_res;
        d.n_units = (int)R_eff;
        const int ns = res_splits(c, R_eff, n_q, S_ring > 0);
        d.n_splits = ns;
        d.split_base = split_base;
        KVS_CK(kv, cudaEventRecord(kv->ev_fork, s));
        KVS_CK(kv, cudaStreamWaitEvent(rstream, kv->ev_fork, 0));
        // Stream capture: the copy stream joins a capture once, from the
        // caller's stream; events recorded outside the current capture are not
        // waited on (the graph runs after all earlier work on the caller's
        // stream, and every earlier ring copy is consumed before its merge).
        // After a capture, the first plain call orders the copy stream after
        // the caller's stream once, since events recorded inside a capture
        // carry no ordering outside it.
        if (cap) {
            if (kv->cs_cap != cap && S_ring > 0) {
                KVS_CK(kv, cudaStreamWaitEvent(kv->cs, kv->ev_fork, 0));
                kv->cs_cap = cap;
            }
            kv->capture_seen = true;
        } else if (kv->capture_seen) {
            KVS_CK(kv, cudaStreamWaitEvent(kv->cs, kv->ev_fork, 0));
            kv->capture_seen = false;
            kv->cs_cap = 0;
            for (int gi = 0; gi < kv->n_groups; ++gi)
                if (kv->free_cap[gi]) kv->free_valid[gi] = 0;
            // a history write last recorded inside a capture ran on the
            // caller's stream before this call, so the wait above covers it
            // (its event may not be waited on outside the capture)
            for (int li = 0; li < c.n_layers; ++li)
                if (kv->hist_cap[li]) {
                    kv->hist_cap[li] = 0;
                    kv->layers[li].pending_min_page = INT_MAX;
                }
        }
        if (tc && S_ring > 0) {
            // launches of res_splits CTAs of kResCtaStages raw stages each, in
            // page order on the resident stream; later ones fold their partials
            // into the first one's records (the first is the widest)
            const long per_launch = ns * kResCtaStages;  // raw stages = 2 per page; even
            for (long st0 = 0; st0 < 2 * R_eff; st0 += per_launch) {
                const long n_st = std::min(per_launch, 2 * R_eff - st0);
                d.slot0 = (int)((first_res + st0 / 2) % R);
                d.page0 = (int)(first_res + st0 / 2);
                d.n_units = (int)(n_st / 2);
                d.n_splits = (int)std::min<long>(ns, n_st);
                d.accumulate = st0 > 0 ? 1 : 0;
                TimedScope ts(kv, rstream, kTChunkMma, (uint64_t)(n_st / 2) * kv->page_bytes);
                KVS_CK(kv, launch_chunk_mma(d, lres.map, d.n_splits, rstream));
                kv->stats.kernel_launches++;
            }
            d.accumulate = 0;
        } else {
            TimedScope ts(kv, rstream, tc ? kTChunkMma : kTDecodeRes, (uint64_t)R_eff * kv->page_bytes);
            KVS_CK(kv, tc ? launch_chunk_mma(d, lres.map, ns, rstream) : launch_decode(d, lres.map, ns, rstream));
            kv->stats.kernel_launches++;
        }
        split_base += ns;
        kv->stats.bytes_resident_read += (uint64_t)R_eff * kv->page_bytes;
    }
    KVS_CK(kv, cudaEventRecord(kv->ev_res, rstream));
    // 2a) zero-copy share: the decode kernel reads streamed pages [S_ring, S)
    //     in place from the mapped pinned history over PCIe, on its own
    //     stream, while the copy engine brings pages [0, S_ring) through the
    //     ring below
    if (S_zc > 0) {
        KVS_CK(kv, cudaStreamWaitEvent(zstream, kv->ev_fork, 0));
        d.region = kv->host_dev + (size_t)layer * kv->P_max * kv->page_bytes;
        d.region_slot_base = 0;
        d.region_slots = (int)kv->P_max;
        d.slot0 = (int)S_ring;
        d.page0 = (int)S_ring;
        d.n_units = (int)S_zc;
        const int ns = zc_splits(c, S_zc, n_q);
        d.n_splits = ns;
        d.split_base = split_base;
        {
            TimedScope ts(kv, zstream, tc ? kTChunkZc : kTDecodeZc, (uint64_t)S_zc * kv->page_bytes);
            KVS_CK(kv, tc ? launch_chunk_mma_zero_copy(d, &kv->map_res, ns, zstream)
                          : launch_decode_zero_copy(d, &kv->map_res, ns, zstream));
        }
        KVS_CK(kv, cudaEventRecord(kv->ev_zc, zstream));
        kv->stats.kernel_launches++;
        split_base += ns;
        kv->stats.pages_streamed += S_zc;
        kv->stats.bytes_h2d += (uint64_t)S_zc * kv->page_bytes;
    }
    // 2b) streamed pages [0, S_ring) through the ring, in ascending page order
    if (S_ring > 0) {
        if (c.n_ring_slots == 0) return fail(kv, KVS_E_INVAL, "internal: streamed pages without a ring");
        if (ls.hist_recorded && ls.pending_min_page < S_ring) {
            if (kv->hist_cap[layer] == cap) KVS_CK(kv, cudaStreamWaitEvent(kv->cs, kv->ev_hist[layer], 0));
            ls.pending_min_page = INT_MAX;
        }
        const int chunk = c.chunk_pages;
        KVS_CK(kv, cudaStreamWaitEvent(xstream, kv->ev_fork, 0));
        // tensor-core ring launches run in order on one stream and fold their
        // partials into the records of the first one
        const int ring_base = split_base;
        int ring_width = 0;
        kv->ring_ctr += (uint64_t)plan_ring(c, n_q, S_ring, (long long)kv->ring_ctr, kv->ring_plan);
        for (const RingCopy& rc : kv->ring_plan) {
            const long i0 = rc.page0;
            const int cpages = rc.pages;
            const int gidx = rc.slot0 / chunk;
            if (rc.new_group && kv->free_valid[gidx] && kv->free_cap[gidx] == cap)
                KVS_CK(kv, cudaStreamWaitEvent(kv->cs, kv->ev_free[gidx], 0));
            uint8_t* dst = kv->ring + (size_t)rc.slot0 * kv->page_bytes;
            const uint8_t* src = kv->host + ((size_t)layer * kv->P_max + (size_t)i0) * kv->page_bytes;
            KVS_CK(kv, cudaMemcpyAsync(dst, src, (size_t)cpages * kv->page_bytes, cudaMemcpyHostToDevice, kv->cs));
            KVS_CK(kv, cudaEventRecord(kv->ev_full[gidx], kv->cs));
            KVS_CK(kv, cudaStreamWaitEvent(xstream, kv->ev_full[gidx], 0));
            // the merge follows the last ring launch on its stream: order it
            // after the resident splits now, while this launch waits for its
            // copy anyway (the resident launches end long before)
            if (i0 + cpages == S_ring) KVS_CK(kv, cudaStreamWaitEvent(xstream, kv->ev_res, 0));
            d.region = kv->ring;
            d.region_slot_base = 0;
            d.region_slots = c.n_ring_slots;
            d.slot0 = rc.slot0;
            d.page0 = (int)i0;
            d.n_units = cpages;
            const int ns = ring_splits(c, n_q, cpages);
            d.n_splits = ns;
            d.split_base = tc ? ring_base : split_base;
            d.accumulate = (tc && i0 > 0) ? 1 : 0;
            {
                TimedScope ts(kv, xstream, tc ? kTChunkMma : kTDecodeRing, (uint64_t)cpages * kv->page_bytes);
                KVS_CK(kv, tc ? launch_chunk_mma(d, &kv->map_ring, ns, xstream)
                              : launch_decode(d, &kv->map_ring, ns, xstream));
            }
            d.accumulate = 0;
            kv->stats.kernel_launches++;
            KVS_CK(kv, cudaEventRecord(kv->ev_free[gidx], xstream));
            kv->free_valid[gidx] = 1;
            kv->free_cap[gidx] = cap;
            if (tc) ring_width = std::max(ring_width, ns);
            else split_base += ns;
            kv->stats.pages_streamed += cpages;
            kv->stats.bytes_h2d += (uint64_t)cpages * kv->page_bytes;
            kv->stats.h2d_copies++;
        }
        split_base += ring_width;
    }

    // 3) log-sum-exp merge of all splits, after the resident (and in-place)
    //    splits; with a ring it runs right behind the last ring launch on its
    //    stream, and the caller's stream waits for it
    cudaStream_t mstream = S_ring > 0 ? xstream : s;
    if (S_ring == 0) KVS_CK(kv, cudaStreamWaitEvent(s, kv->ev_res, 0));
    if (S_zc > 0) KVS_CK(kv, cudaStreamWaitEvent(mstream, kv->ev_zc, 0));
    MergeArgs m;
    m.part = kv->part;
    m.n_splits = split_base;
    m.n_rows = rows;
    m.out = dout;
    m.lse = dlse;
    m.err = nullptr;  // a timed-out wait is reported by kvs_sync / kvs_get_stats
    {
        TimedScope ts(kv, mstream, kTMerge, 0);
        KVS_CK(kv, launch_merge(m, mstream));
    }
    kv->stats.kernel_launches++;
    if (mstream != s) {
        KVS_CK(kv, cudaEventRecord(kv->ev_ring, mstream));
        KVS_CK(kv, cudaStreamWaitEvent(s, kv->ev_ring, 0));
    }
    if (host_out)
        KVS_CK(kv, cudaMemcpyAsync(out, dout, (size_t)rows * kHeadDim * 4, cudaMemcpyDeviceToHost, s));
    if (host_lse) KVS_CK(kv, cudaMemcpyAsync(lse, dlse, (size_t)rows * 4, cudaMemcpyDeviceToHost, s));
    kv->stats.attends++;
    return KVS_OK;
}

int kvs_export_page(kvs_t* kv, int layer, int page, int from_device, void* host_dst) {
    if (!kv || !host_dst) return fail(kv, KVS_E_INVAL, "null argument");
    const kvs_config& c = kv->cfg;
    if (layer < 0 || layer >= c.n_layers || page < 0 || page >= kv->P_max)
        return fail(kv, KVS_E_INVAL, "layer/page out of range");
    std::vector<uint8_t> buf(kv->page_bytes);
    if (from_device) {
        if (aux_layer(kv, layer) && !kv->draft_active)
            return fail(kv, KVS_E_INVAL, "auxiliary layers are ejected: no resident pages");
        int kind, idx;
        plan_page_r(layer_res(kv, layer).R, kv->layers[layer].len, page, &kind, &idx);
        if (kind != KVS_PAGE_RESIDENT) return fail(kv, KVS_E_INVAL, "page is not resident");
        DeviceGuard g(kv->device);
        const uint8_t* src = layer_res(kv, layer).base + (size_t)idx * kv->page_bytes;
        KVS_CK(kv, cudaMemcpy(buf.data(), src, kv->page_bytes, cudaMemcpyDeviceToHost));
    } else {
        std::memcpy(buf.data(), kv->host + ((size_t)layer * kv->P_max + page) * kv->page_bytes, kv->page_bytes);
    }
    uint8_t* out = static_cast<uint8_t*>(host_dst);
    const int H = c.n_kv_heads;
    // canonical V block: fp16 d, [fp16 m], [fifth-bit word], codes
    int vblk = 0, off_vh = 0, off_vd = 0, off_vm = 0;
    bool has_h = false, has_m = false;
    switch (c.type_v) {
#define KVS_V_FIELDS(T)                                                               \
    vblk = PageGeom<T>::kVBlockBytes; off_vh = PageGeom<T>::kOffVh;                   \
    off_vd = PageGeom<T>::kOffVd; off_vm = PageGeom<T>::kOffVm;                      \
    has_h = PageGeom<T>::kVhRow > 0; has_m = PageGeom<T>::kVmRow > 0;
        case KVS_TYPE_Q8_0: KVS_V_FIELDS(kVQ8_0) break;
        case KVS_TYPE_Q5_0: KVS_V_FIELDS(kVQ5_0) break;
        case KVS_TYPE_Q4_1: KVS_V_FIELDS(kVQ4_1) break;
        case KVS_TYPE_Q5_1: KVS_V_FIELDS(kVQ5_1) break;
        case KVS_TYPE_F16: KVS_V_FIELDS(kVF16) break;
        default: KVS_V_FIELDS(kVQ4_0) break;
#undef KVS_V_FIELDS
    }
    const bool v8 = c.type_v == KVS_TYPE_Q8_0;
    const bool k16 = c.type_k == KVS_TYPE_F16;
    // V fields follow K: 34,816 B in for Q8_0 K, 65,536 B for f16 K
    const int off_vq = k16 ? PageGeom<kVF16, kKF16>::kOffVq : PageGeom<kVQ4_0>::kOffVq;
    const int phb = page_head_bytes(c.type_v, c.type_k);
    const int kblk = k16 ? 64 : 34;  // canonical K block: Q8_0, or the 32 fp16 values
    uint8_t* kout = out;
    uint8_t* vout = out + (size_t)kPageTokens * H * kBlocks * kblk;
    for (int t = 0; t < kPageTokens; ++t)
        for (int h = 0; h < H; ++h) {
            const uint8_t* ph = buf.data() + (size_t)h * phb;
            for (int b = 0; b < kBlocks; ++b) {
                uint8_t* kb = kout + (((size_t)t * H + h) * kBlocks + b) * kblk;
                if (k16) {
                    std::memcpy(kb, ph + t * (kHeadDim * 2) + b * 64, 64);
                } else {
                    std::memcpy(kb, ph + kOffKd + t * 8 + b * 2, 2);
                    std::memcpy(kb + 2, ph + kOffKq + t * kHeadDim + b * 32, 32);
                }
                uint8_t* vb = vout + (((size_t)t * H + h) * kBlocks + b) * vblk;
                if (c.type_v == KVS_TYPE_F16) {  // the 32 values of the block
                    std::memcpy(vb, ph + off_vq + t * (kHeadDim * 2) + b * 64, 64);
                    continue;
                }
                std::memcpy(vb, ph + off_vd + t * 8 + b * 2, 2);
                int at = 2;
                if (has_m) { std::memcpy(vb + at, ph + off_vm + t * 8 + b * 2, 2); at += 2; }
                if (has_h) { std::memcpy(vb + at, ph + off_vh + t * 16 + b * 4, 4); at += 4; }
                if (v8) std::memcpy(vb + at, ph + off_vq + t * kHeadDim + b * 32, 32);
                else std::memcpy(vb + at, ph + off_vq + t * 64 + b * 16, 16);
            }
        }
    return KVS_OK;
}

int kvs_page_location(kvs_t* kv, int layer, int page, int* kind, int* index) {
    if (!kv || !kind || !index) return fail(kv, KVS_E_INVAL, "null argument");
    if (layer < 0 || layer >= kv->cfg.n_layers) return fail(kv, KVS_E_INVAL, "layer out of range");
    if (aux_layer(kv, layer) && !kv->draft_active)
        return fail(kv, KVS_E_INVAL, "auxiliary layers are ejected: no resident pages");
    return plan_page_r(layer_res(kv, layer).R, kv->layers[layer].len, page, kind, index);
}

int kvs_layer_length(kvs_t* kv, int layer, int* n_tokens) {
    if (!kv || !n_tokens || layer < 0 || layer >= kv->cfg.n_layers) return fail(kv, KVS_E_INVAL, "bad argument");
    *n_tokens = kv->layers[layer].len;
    return KVS_OK;
}

int kvs_get_config(kvs_t* kv, kvs_config* out) {
    if (!kv || !out) return fail(kv, KVS_E_INVAL, "null argument");
    *out = kv->cfg;
    return KVS_OK;
}

int kvs_get_stats(kvs_t* kv, kvs_stats* out) {
    if (!kv || !out) return fail(kv, KVS_E_INVAL, "null argument");
    if (!kv->timed.empty()) {
        DeviceGuard g(kv->device);
        int rc = wait_event(kv, kv->timed.back().b, 120.0);
        if (rc != KVS_OK) return rc;
        fold_timed(kv);
    }
    *out = kv->stats;
    return KVS_OK;
}

int kvs_reset_stats(kvs_t* kv) {
    if (!kv) return fail(kv, KVS_E_INVAL, "null handle");
    if (!kv->timed.empty()) {
        DeviceGuard g(kv->device);
        int rc = wait_event(kv, kv->timed.back().b, 120.0);
        if (rc != KVS_OK) return rc;
        fold_timed(kv);
    }
    kv->stats = kvs_stats{};
    return KVS_OK;
}

int kvs_set_zero_copy_pct(kvs_t* kv, int pct, int pct_wide) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    if (pct < -1 || pct > 100 || pct_wide < -1 || pct_wide > 100)
        return fail(kv, KVS_E_INVAL, fmt("in-place shares %d / %d outside -1..100", pct, pct_wide));
    // the partial buffer is sized for every share
    if (pct >= 0) kv->cfg.zero_copy_pct = pct;
    if (pct_wide >= 0) kv->cfg.zero_copy_pct_wide = pct_wide;
    return KVS_OK;
}

int kvs_phase_layout(const kvs_config* resolved, int width, size_t pinned_bytes, int draft_active,
                     kvs_arena_status* out) {
    if (!resolved || !out) { g_last_error = "kvs_phase_layout: null argument"; return KVS_E_INVAL; }
    const kvs_config& c = *resolved;
    if (!(c.flags & KVS_FLAG_PHASE_ARENA) || c.arena_bytes == 0) {
        g_last_error = "kvs_phase_layout: the config is not a resolved phase arena";
        return KVS_E_INVAL;
    }
    if (width < 1 || width > c.max_q_tokens) {
        g_last_error = fmt("kvs_phase_layout: width %d outside 1..max_q_tokens (%d)", width, c.max_q_tokens);
        return KVS_E_INVAL;
    }
    kvs_config cw = c;
    cw.max_q_tokens = width;
    const size_t aux_bytes = (draft_active && c.n_aux_layers > 0) ? aux_region_bytes(c) : 0;
    const long R = aux_bytes + pinned_bytes < c.arena_bytes
                       ? resident_fit(cw, c.arena_bytes - aux_bytes - pinned_bytes, pages_for(c.max_ctx))
                       : 0;
    if (R < 1) {
        g_last_error = "kvs_phase_layout: no resident page fits";
        return KVS_E_ARENA;
    }
    fill_status(c, R, width, c.arena_bytes, pinned_bytes, draft_active != 0,
                width == c.max_q_tokens ? KVS_PHASE_PREFILL : KVS_PHASE_DECODE, out);
    return KVS_OK;
}

int kvs_set_phase(kvs_t* kv, int phase, int width, void* stream) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    if (!kv->phase_arena) return fail(kv, KVS_E_INVAL, "no phase arena (arena_bytes with n_resident_pages = 0)");
    if (phase == KVS_PHASE_PREFILL) {
        if (width == 0) width = kv->cfg.max_q_tokens;
    } else if (phase == KVS_PHASE_DECODE) {
        if (width == 0) width = 1;
    } else {
        return fail(kv, KVS_E_INVAL, fmt("unknown phase %d", phase));
    }
    if (width < 1 || width > kv->cfg.max_q_tokens)
        return fail(kv, KVS_E_INVAL, fmt("phase width %d outside 1..max_q_tokens (%d)", width, kv->cfg.max_q_tokens));
    DeviceGuard g(kv->device);
    const int rc = relayout(kv, width, kv->pin_bytes, kv->draft_active, static_cast<cudaStream_t>(stream));
    if (rc == KVS_OK) kv->phase = phase;
    return rc;
}

int kvs_pin(kvs_t* kv, size_t bytes, void** dev_ptr, void* stream) {
    if (!kv || !dev_ptr || bytes == 0) return fail(kv, KVS_E_INVAL, "kvs_pin: bad argument");
    if (!kv->phase_arena) return fail(kv, KVS_E_INVAL, "no phase arena (arena_bytes with n_resident_pages = 0)");
    if (!kv->draft_active) return fail(kv, KVS_E_INVAL, "the draft is ejected: nothing can be pinned");
    const size_t total = kv->pin_bytes + align_up(bytes);
    DeviceGuard g(kv->device);
    const int rc = relayout(kv, kv->width, total, true, static_cast<cudaStream_t>(stream));
    if (rc != KVS_OK) return rc;
    const size_t aux_bytes = kv->cfg.n_aux_layers > 0 ? aux_region_bytes(kv->cfg) : 0;
    *dev_ptr = kv->arena + kv->alloc_bytes - aux_bytes - total;
    return KVS_OK;
}

int kvs_draft_eject(kvs_t* kv, void* stream) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    if (!kv->phase_arena) return fail(kv, KVS_E_INVAL, "no phase arena (arena_bytes with n_resident_pages = 0)");
    if (!kv->draft_active) return KVS_OK;
    DeviceGuard g(kv->device);
    return relayout(kv, kv->width, 0, false, static_cast<cudaStream_t>(stream));
}

int kvs_draft_restore(kvs_t* kv, void* stream) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    if (!kv->phase_arena) return fail(kv, KVS_E_INVAL, "no phase arena (arena_bytes with n_resident_pages = 0)");
    if (kv->draft_active) return KVS_OK;
    DeviceGuard g(kv->device);
    return relayout(kv, kv->width, 0, true, static_cast<cudaStream_t>(stream));
}

int kvs_get_arena(kvs_t* kv, kvs_arena_status* out) {
    if (!kv || !out) return fail(kv, KVS_E_INVAL, "null argument");
    fill_status(kv->cfg, kv->cfg.n_resident_pages, kv->width, kv->alloc_bytes, kv->pin_bytes, kv->draft_active,
                kv->phase, out);
    return KVS_OK;
}

int kvs_set_profiling(kvs_t* kv, int enable) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    if (enable) kv->cfg.flags |= KVS_FLAG_PROFILE;
    else kv->cfg.flags &= ~KVS_FLAG_PROFILE;
    return KVS_OK;
}

int kvs_sync(kvs_t* kv, void* stream, double timeout_s) {
    if (!kv) return fail(nullptr, KVS_E_INVAL, "null handle");
    DeviceGuard g(kv->device);
    return sync_all(kv, static_cast<cudaStream_t>(stream), timeout_s);
}

int kvs_measure_h2d(kvs_t* kv, size_t chunk_bytes, size_t total_bytes, int reps, double* gbs) {
    if (!kv || !gbs || chunk_bytes == 0 || reps < 1) return fail(kv, KVS_E_INVAL, "bad argument");
    uint8_t* dst = kv->cfg.n_ring_slots ? kv->ring : kv->resident;
    const size_t dst_bytes = kv->cfg.n_ring_slots ? (size_t)kv->cfg.n_ring_slots * kv->page_bytes
                                                  : (size_t)target_layers(kv->cfg) * kv->cfg.n_resident_pages * kv->page_bytes;
    if (chunk_bytes > dst_bytes) return fail(kv, KVS_E_INVAL, "chunk larger than the device region");
    total_bytes = std::min(total_bytes, kv->host_bytes) / chunk_bytes * chunk_bytes;
    if (total_bytes == 0) return fail(kv, KVS_E_INVAL, "total smaller than one chunk");
    DeviceGuard g(kv->device);
    KVS_CK(kv, cudaStreamSynchronize(kv->cs));
    cudaEvent_t a, b;
    KVS_CK(kv, cudaEventCreate(&a));
    KVS_CK(kv, cudaEventCreate(&b));
    double best = 0.0;
    const size_t slots = dst_bytes / chunk_bytes;
    for (int r = 0; r < reps; ++r) {
        cudaEventRecord(a, kv->cs);
        for (size_t off = 0, i = 0; off < total_bytes; off += chunk_bytes, ++i)
            cudaMemcpyAsync(dst + (i % slots) * chunk_bytes, kv->host + off, chunk_bytes,
                            cudaMemcpyHostToDevice, kv->cs);
        cudaEventRecord(b, kv->cs);
        int rc = wait_event(kv, b, 120.0);
        if (rc != KVS_OK) { cudaEventDestroy(a); cudaEventDestroy(b); return rc; }
        float ms = 0;
        cudaEventElapsedTime(&ms, a, b);
        best = std::max(best, total_bytes / (ms * 1e-3) / 1e9);
    }
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    *gbs = best;
    return KVS_OK;
}

int kvs_selftest_bounded_wait(int device, double limit_s, int* err_bits) {
    if (!err_bits || limit_s <= 0 || limit_s > 10) return fail(nullptr, KVS_E_INVAL, "bad argument");
    int n_dev = 0;
    if (cudaGetDeviceCount(&n_dev) != cudaSuccess || device < 0 || device >= n_dev) {
        cudaGetLastError();
        return fail(nullptr, KVS_E_INVAL, "no such CUDA device");
    }
    DeviceGuard g(device);
    int* d_err = nullptr;
    KVS_CK(nullptr, cudaMalloc(reinterpret_cast<void**>(&d_err), sizeof(int)));
    cudaStream_t st = nullptr;
    cudaEvent_t done = nullptr;
    int rc = KVS_OK;
    if (cudaMemset(d_err, 0, sizeof(int)) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&done, cudaEventDisableTiming) != cudaSuccess ||
        launch_wait_selftest(d_err, (uint64_t)(limit_s * 1e9), st) != cudaSuccess ||
        cudaEventRecord(done, st) != cudaSuccess) {
        rc = fail(nullptr, KVS_E_CUDA, "self-test launch failed");
    } else {
        rc = wait_event(nullptr, done, limit_s + 30.0);
        if (rc == KVS_OK && cudaMemcpy(err_bits, d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
            rc = fail(nullptr, KVS_E_CUDA, "self-test readback failed");
    }
    if (done) cudaEventDestroy(done);
    if (st) cudaStreamDestroy(st);
    cudaFree(d_err);
    return rc;
}

const char* kvs_last_error(kvs_t* kv) {
    if (kv) return kv->err.c_str();
    return g_last_error.c_str();
}

}  // extern "C"

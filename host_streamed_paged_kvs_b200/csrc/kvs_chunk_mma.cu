// kvs_chunk_mma.cu -- K4: multi-token attention over quantized pages on the
// 5th-generation tensor cores (tcgen05), for speculative-verify batches and
// prefill chunks ("llama.cpp adaptive KV streaming - spec fork notes", Phase
// arena: speculative verify batches of 1 + n_draft tokens; 256-token ubatches
// on "RaymondHuang210129/llama.cpp-adaptive-kv-streaming", Summary).
//
// CTA = (split, kv head, pair of 128-row M tiles of the head's n_q x G query
// rows): both tiles share every dequantized K/V sub-stage, so the producers'
// work and the shared-memory operand traffic they cause are paid once per two
// tiles, and the tensor cores alternate between the tiles' products while
// each tile's softmax runs.  512 threads in four warp-specialized roles on
// 64-key sub-stages, handing work to each other only through mbarriers:
//
//   softmax warps 0..3 (tile 0) and 4..7 (tile 1), thread = query row = TMEM
//     lane, whole 64-key rows: put the tile's Q into tensor memory once,
//     staged through the K^/V^ operand buffers, and report it on the tile's Q
//     barrier (the loads start without waiting for Q; the producers' first
//     operand write and the tile's first S wait for it), then
//     per sub-stage read S, apply the causal mask and the 1/sqrt(128) scale in
//     the log2 domain, keep a per-row reference max that only moves when the
//     row max exceeds it by more than 2^8 (then rescale the row of O in TMEM),
//     and write P in fp16 over the S columns just read;
//   producer warps 8, 9, 11, 12 and 13
//     dequantize each 64-key half of a raw Q8_0/Q4_0 stage (128 keys, landed
//     by TMA, three raw stages in flight where shared memory allows, else two)
//     into fp16 UMMA operand tiles with the 128-byte swizzle:
//       K^ = d*q8 as [keys][dims] (K-major), split into hi = fp16(d*q8) and
//       lo = fp16(d*q8 - hi) so the scores carry no fp16 rounding of K
//       (two buffers, free again once both tiles' S MMAs that read them
//       complete);
//       V^ = fp16(d*(q4-8)) as [keys][dims] (read as an MN-major B operand;
//       three buffers, free again once both tiles' PV MMAs complete);
//   MMA warps 10 (tile 0) and 15 (tile 1), one lane each
//     poll the barriers without blocking and issue, whichever is ready
//     first: S_t = Q_t K^_hi^T + Q_t K^_lo^T (tcgen05.mma M=128 N=64 K=16,
//     A = Q_t from tensor memory, fp32 accumulate) of tile t once the K^
//     buffer is full, it is the tile's turn (the tiles' S products alternate,
//     so one tile's softmax overlaps the other's products instead of both
//     running at once) and the tile's previous PV product has been issued (P_t
//     lives in the S_t columns; the tensor cores run the MMAs in issue order);
//     and O_t += P_t V^ (M=128 N=128 K=16, A = P_t from tensor memory) once
//     the softmax wrote P_t and V^ is written, with the tile's next S right
//     behind it.  Only the B operands (K^, V^) are read from shared memory;
//   load warp 14 (one lane)
//     issues each raw stage (a TMA tile of the K quants, bulk copies of the
//     other fields) as soon as the producers release its buffer, so the loads
//     never wait behind the MMA issue.
//
// Tensor memory (512 columns, one CTA per SM), per tile t at 256 t: O_t (128
// fp32 columns) at +0, S_t (64) at +128 with P_t (fp16 pairs, 32) over its
// first half, Q_t (fp16 pairs, 64) at +192.
// At the end O, m, l of every valid row are written as the split's partials
// for the LSE merge, each warp's 32 rows staged in shared memory so that a
// record row (and the previous record folded into it) moves as whole 128-byte
// lines.  No cluster, no multicast.
//
// Warp w issues on sub-partition w mod 4 of the SM, and the arithmetic of the
// other warps there delays the tensor-core issue of an MMA warp on the same
// sub-partition (each sub-partition holds two softmax warps: the lane
// quarter a warp may read from tensor memory is w mod 4).  So each tile has
// its own MMA warp, on sub-partitions 2 and 3, and the producers run on the
// others but one (warp 11).
#include <cuda_fp16.h>
#include <math_constants.h>

#include <atomic>

#include "kvs_internal.h"
#include "kvs_ptx.cuh"

namespace kvs {
namespace {

constexpr int kTiles = 2;                                   // M tiles per CTA
constexpr int kTileWarps = 4;                               // softmax warps per tile
constexpr int kSoftWarps = kTiles * kTileWarps;             // 8
constexpr int kProdWarps = 5;                               // warps 8, 9, 11, 12, 13
constexpr int kMmaWarp0 = 10;                               // tile 0's products, sub-partition 2
constexpr int kMmaWarp1 = 15;                               // tile 1's products, sub-partition 3
constexpr int kLoadWarp = 14;                               // sub-partition 2, beside MMA warp 0
constexpr int kTcThreads = (kSoftWarps + kProdWarps + 3) * 32;  // 512
static_assert(kMmaWarp0 % 4 != kMmaWarp1 % 4 && kMmaWarp0 % 4 == kLoadWarp % 4 && kTcThreads == 512,
              "one MMA warp per tile on two sub-partitions");
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kMTile = 128;
constexpr int kRawKeys = 128;  // keys per raw (TMA) stage
constexpr int kSubKeys = 64;   // keys per dequant / MMA sub-stage
constexpr int kRawKq = 0;
constexpr int kMaxRawStages = 3;  // raw stages in flight: three where they fit, else two
constexpr int kKBufs = 2;
constexpr int kVBufs = 3;
constexpr int kKVBytes = kSubKeys * kHeadDim * 2;     // 16384: K^hi, K^lo or V^ [64][128] fp16
// barriers: raw_full[3] raw_free[3] k_full[2] k_free[2] v_full[3] v_free[3]
//           s_full[tile] p_full[tile] o_free[tile] q_full[tile]
constexpr int kBarK = 2 * kMaxRawStages;           // 6
constexpr int kBarV = kBarK + 2 * kKBufs;          // 10
constexpr int kBarT = kBarV + 2 * 3;               // 16
constexpr int kNumBars = kBarT + 4 * kTiles;       // 24
constexpr uint32_t kTmemCols = 512;
// columns within a tile's 256: O, S (P over its first 32 columns), Q
constexpr uint32_t kTileCols = 256, kColO = 0, kColS = 128, kColQ = 192;
static_assert(kKVBytes % 1024 == 0, "swizzled tiles need 1024-B alignment");

// Raw-stage and shared-memory layout by V type.  Raw stage (128 keys, as the
// pages hold them): Kq [128][128] @ 0, Kd @ 16384, Vq @ 17408 (64 B per key
// for Q4_0 and Q5_0 V, 128 B for Q8_0 V, 256 B of values for F16 V), the Q5_x
// fifth bits (16 B per key), Vd (none for F16), then the Q4_1 / Q5_1 minima
// (8 B per key).  Shared memory: three raw stages where they fit (else two),
// then [2] x (K^hi | K^lo), [3] x V^, the barriers, the TMEM slot, the abort
// flag and the tiles' S turn counters (Q4_0 V: K^ @ 79872, V^ @ 145408,
// barriers @ 194560).  The K^/V^ buffers also stage Q before the first
// operand is written, and the raw stages the epilogue's record rows.
// f16 K (the f16-f16 pair): the raw stage holds each key's values as two
// 128-byte rows (dims 0..63, 64..127) and K^ needs no lo tile.
template <int VT, int KT = kKQ8_0>
struct TcGeom {
    using PG = PageGeom<VT, KT>;
    static constexpr int kKRows = kRawKeys * PG::kKqRow / 128;                  // 128-byte K rows per raw stage
    static constexpr int kRawKd = kRawKeys * PG::kKqRow;                         // 16384 for Q8_0 K
    static constexpr int kRawVq = kRawKd + kRawKeys * PG::kKdRow;                // 17408 for Q8_0 K
    static constexpr int kRawVh = kRawVq + kRawKeys * PG::kVqRow;                // Q5_x fifth bits
    static constexpr int kRawVd = kRawVh + kRawKeys * PG::kVhRow;
    static constexpr int kRawVm = kRawVd + kRawKeys * PG::kVdRow;                // Q4_1 / Q5_1 minima
    static constexpr int kRawBytes = kRawVm + kRawKeys * PG::kVmRow;
    static constexpr int kKHalves = KT == kKF16 ? 1 : 2;                         // K^ tiles per buffer
    // the dequantized tiles, barriers and slack; three raw stages where they fit
    static constexpr size_t kRest = (size_t)(kKBufs * kKHalves + kVBufs) * kKVBytes + kNumBars * 8 + 1024 + 32;
    static constexpr int kRawStages = (size_t)kMaxRawStages * kRawBytes + kRest <= 232448 ? kMaxRawStages : 2;
    static constexpr size_t kOffK = (size_t)kRawStages * kRawBytes;
    static constexpr size_t kOffV = kOffK + kKBufs * kKHalves * kKVBytes;
    static constexpr size_t kOffBar = kOffV + kVBufs * kKVBytes;
    static constexpr size_t kOffTmem = kOffBar + kNumBars * 8;
    static constexpr size_t kOffAbort = kOffTmem + 4;
    static constexpr size_t kOffTurn = kOffTmem + 8;  // S batches issued, per tile
    static constexpr size_t kSmem = 1024 + kOffTmem + 16;
    static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kRawBytes % 1024 == 0,
                  "swizzled tiles need 1024-B alignment");
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert((size_t)kSoftWarps * 32 * 272 <= (size_t)(kKBufs * kKHalves + kVBufs) * kKVBytes,
                  "the softmax warps' Q staging fits the operand buffers");
};
static_assert(TcGeom<kVQ4_0>::kRawStages == 3 && TcGeom<kVQ8_0>::kRawStages == 3 && TcGeom<kVF16>::kRawStages == 2,
              "raw stages in flight");
static_assert(TcGeom<kVQ5_0>::kRawBytes == 28672, "Q5_0 raw stage");
static_assert(TcGeom<kVQ4_1>::kRawBytes == 27648 && TcGeom<kVQ5_1>::kRawBytes == 29696, "Q4_1 / Q5_1 raw stages");
static_assert(TcGeom<kVF16>::kRawBytes == 50176, "F16 raw stage");
static_assert(TcGeom<kVF16, kKF16>::kRawBytes == 65536, "f16-f16 raw stage");

// instruction descriptors: f16 x f16 -> f32, M = 128; A K-major;
// S: N = 64, B K-major; PV: N = 128, B MN-major
constexpr uint32_t kIdescS = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// byte offset of element (row, col) of a fp16 tile of `rows` rows stored in
// 64-column halves (rows * 128 B each), rows of 128 B in 8-row groups of 1 KB,
// 16-byte chunks XOR-swizzled by the row within its group (128-byte swizzle)
__device__ __forceinline__ uint32_t tile_off(int rows, int row, int col) {
    return (uint32_t)((col >> 6) * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
                      ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}

// shared-memory matrix descriptor (version 1, 128-byte swizzle)
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((start >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand of `rows` rows, k-step kk of 16 elements
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int rows, int kk) {
    return smem_desc(base + (kk >> 2) * rows * 128 + (kk & 3) * 32, 16, 1024);
}
// MN-major operand V^ [64 keys][128 dims]: 8-key groups 1 KB apart (K
// direction), 64-dim halves 8 KB apart (N direction); k-step kk = keys 16kk..
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int kk) {
    return smem_desc(base + kk * 2048, kSubKeys * 128, 1024);
}

__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// 2^x with the hardware approximation (flush-to-zero; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// packed pairs of fp32 (one instruction for two lanes of arithmetic)
__device__ __forceinline__ unsigned long long f2_bits(float2 v) {
    return (unsigned long long)__float_as_uint(v.x) | ((unsigned long long)__float_as_uint(v.y) << 32);
}
__device__ __forceinline__ float2 bits_f2(unsigned long long b) {
    return make_float2(__uint_as_float((uint32_t)b), __uint_as_float((uint32_t)(b >> 32)));
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {  // a * b + c, each lane rounded once
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
    return bits_f2(r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return bits_f2(r);
}

// D (+)= A B with A (M=128 rows, 16-bit pairs per column) read from tensor memory
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
    float f[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
    tmem_st32(taddr, f);
}

// non-blocking probe of an mbarrier phase
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Q5_0 V: bit 4 of the codes of dims j and j + 1 of a block (bits j, j + 1 of
// its fifth-bit word hw), placed at bit 4 of the low and high fp16 halves
__device__ __forceinline__ uint32_t fifth_bits(uint32_t hw, int j) {
    return (((hw >> j) & 1u) << 4) | (((hw >> (j + 1)) & 1u) << 20);
}


// ZC = true: the raw stages are read in place from mapped pinned host memory
// (the history's device alias) by the load warp's 16-byte asynchronous copies,
// the K quants placed in the swizzle the tensor map would produce.
template <int VT, int KT, bool ZC>
__global__ void __launch_bounds__(kTcThreads, 1)
    chunk_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap) {
    using TG = TcGeom<VT, KT>;
    using PG = PageGeom<VT, KT>;
    constexpr int kRawKd = TG::kRawKd, kKHalves = TG::kKHalves;
    constexpr int kRawVq = TG::kRawVq, kRawVh = TG::kRawVh, kRawVd = TG::kRawVd, kRawBytes = TG::kRawBytes;
    constexpr int kRawVm = TG::kRawVm;
    constexpr size_t kOffK = TG::kOffK, kOffV = TG::kOffV, kOffBar = TG::kOffBar;
    constexpr size_t kOffTmem = TG::kOffTmem, kOffAbort = TG::kOffAbort;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* raw = smem;
    uint8_t* sK = smem + kOffK;
    uint8_t* sV = smem + kOffV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    constexpr int kRS = TG::kRawStages;
    uint64_t* raw_full = bars + 0;                 // [raw stage] TMA bytes landed
    uint64_t* raw_free = bars + kMaxRawStages;     // [raw stage] producers done reading it (6 warp arrivals)
    uint64_t* k_full = bars + kBarK;               // [2] producers wrote K^hi/K^lo (6 warp arrivals)
    uint64_t* k_free = bars + kBarK + 2;           // [2] both tiles' S MMAs reading a K^ buffer complete
    uint64_t* v_full = bars + kBarV;               // [3] producers wrote V^ (6 warp arrivals)
    uint64_t* v_free = bars + kBarV + 3;           // [3] both tiles' PV MMAs reading a V^ buffer complete
    uint64_t* s_full = bars + kBarT;               // [tile] S_t MMA complete
    uint64_t* p_full = bars + kBarT + kTiles;      // [tile] softmax wrote P_t (4 warp arrivals)
    uint64_t* o_free = bars + kBarT + 2 * kTiles;  // [tile] PV_t MMA complete (P_t / S_t columns free)
    uint64_t* q_full = bars + kBarT + 3 * kTiles;  // [tile] softmax wrote Q_t to tensor memory (4 warp arrivals)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
    // set by a thread whose bounded wait gave up; everyone then skips the
    // remaining waits and work (there are no named barriers to leave behind)
    volatile int* sAbort = reinterpret_cast<volatile int*>(smem + kOffAbort);
    // S batches fully issued by each tile's MMA warp: the two tiles take turns
    volatile int* sIssued = reinterpret_cast<volatile int*>(smem + TG::kOffTurn);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const int rows_head = a.n_q * a.group;
    // tiles of this CTA: 2 z and 2 z + 1 (the second one only if it has rows)
    const int n_tiles = ((2 * blockIdx.z + 1) * kMTile < rows_head) ? 2 : 1;
    const int raw0 = (int)(((long)blockIdx.x * 2 * a.n_units) / a.n_splits);  // first raw stage
    const int n_raw = (int)(((long)(blockIdx.x + 1) * 2 * a.n_units) / a.n_splits) - raw0;
    const int n_sub = 2 * n_raw;  // 64-key sub-stages

    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        *sAbort = 0;
        sIssued[0] = 0;
        sIssued[1] = 0;
        for (int k = 0; k < kMaxRawStages; ++k) {
            mbar_init(&raw_full[k], ZC ? 32 : 1);  // in place: one arrival per load lane
            mbar_init(&raw_free[k], kProdWarps);
        }
        for (int k = 0; k < kKBufs; ++k) {
            mbar_init(&k_full[k], kProdWarps);
            mbar_init(&k_free[k], n_tiles);  // one commit per tile's MMA warp
        }
        for (int k = 0; k < kVBufs; ++k) {
            mbar_init(&v_full[k], kProdWarps);
            mbar_init(&v_free[k], n_tiles);
        }
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], kTileWarps);
            mbar_init(&o_free[t], 1);
            mbar_init(&q_full[t], kTileWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = *tmem_slot;
    // softmax warps: tile of this warp, its first TMEM column, the warp's lanes
    const int my_tile = warp / kTileWarps;
    const uint32_t tcol = (uint32_t)my_tile * kTileCols;
    const uint32_t lane_off = (uint32_t)((warp % kTileWarps) * 32) << 16;
    bool ok = true;
    auto fail_wait = [&](uint64_t* bar, uint32_t parity) {  // true if the wait gave up
        if (!ok || *sAbort) { ok = false; return true; }
        if (!mbar_wait_bounded(bar, parity, a.err)) { ok = false; *sAbort = 1; return true; }
        return false;
    };

    if (warp == kLoadWarp) {
        // ============================ load warp ============================
        // raw stage r into buffer r % kRS once the producers released the
        // stage that used it before (r - kRS)
        if (ZC || lane == 0) {
            for (int r = 0; r < n_raw; ++r) {
                const int buf = r % kRS;
                if (r >= kRS && fail_wait(&raw_free[buf], ((r - kRS) / kRS) & 1)) break;
                const int sg = raw0 + r;
                const int u = sg >> 1, half = sg & 1;
                const int slot = (a.slot0 + u) % a.region_slots;
                const uint8_t* ph = a.region + ((size_t)slot * a.n_kv + h) * PG::kHeadBytes;
                uint8_t* dst = raw + buf * kRawBytes;
                uint64_t* b = &raw_full[buf];
                if constexpr (ZC) {
                    // K quants (or f16 K values): 128-byte row kr of the half
                    // page, 16-byte chunk k -> swizzled; the other fields as they lie
                    const uint8_t* kq = ph + PG::kOffKq + half * (kRawKeys * PG::kKqRow);
#pragma unroll 4
                    for (int c = lane; c < TG::kKRows * 8; c += 32) {
                        const int kr = c >> 3, k = c & 7;
                        cp_async16(dst + kRawKq + kr * 128 + ((k ^ (kr & 7)) << 4), kq + kr * 128 + k * 16);
                    }
                    auto copy_field = [&](int dst_off, int src_off, int row_bytes) {
                        const uint8_t* src = ph + src_off + half * (kRawKeys * row_bytes);
                        for (int c = lane; c < kRawKeys * row_bytes / 16; c += 32)
                            cp_async16(dst + dst_off + c * 16, src + c * 16);
                    };
                    if constexpr (PG::kKdRow > 0) copy_field(kRawKd, PG::kOffKd, PG::kKdRow);
                    copy_field(kRawVq, PG::kOffVq, PG::kVqRow);
                    if constexpr (PG::kVhRow > 0) copy_field(kRawVh, PG::kOffVh, PG::kVhRow);
                    if constexpr (PG::kVdRow > 0) copy_field(kRawVd, PG::kOffVd, PG::kVdRow);
                    if constexpr (PG::kVmRow > 0) copy_field(kRawVm, PG::kOffVm, PG::kVmRow);
                    cp_async_arrive(b);
                } else {
                    mbar_expect_tx(b, kRawBytes);
                    const int krow = ((a.region_slot_base + slot) * a.n_kv + h) * PG::kRows + half * TG::kKRows;
#pragma unroll
                    for (int kr = 0; kr < TG::kKRows; kr += 128)  // boxes of 128 rows of 128 B
                        tma_load_2d(dst + kRawKq + kr * 128, &kmap, 0, krow + kr, b);
                    if constexpr (PG::kKdRow > 0)
                        bulk_load(dst + kRawKd, ph + PG::kOffKd + half * (kRawKeys * PG::kKdRow), kRawKeys * PG::kKdRow, b);
                    bulk_load(dst + kRawVq, ph + PG::kOffVq + half * (kRawKeys * PG::kVqRow), kRawKeys * PG::kVqRow, b);
                    if constexpr (PG::kVhRow > 0)
                        bulk_load(dst + kRawVh, ph + PG::kOffVh + half * (kRawKeys * PG::kVhRow), kRawKeys * PG::kVhRow, b);
                    if constexpr (PG::kVdRow > 0)
                        bulk_load(dst + kRawVd, ph + PG::kOffVd + half * (kRawKeys * kBlocks * 2), kRawKeys * kBlocks * 2, b);
                    if constexpr (PG::kVmRow > 0)
                        bulk_load(dst + kRawVm, ph + PG::kOffVm + half * (kRawKeys * PG::kVmRow), kRawKeys * PG::kVmRow, b);
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp0 || warp == kMmaWarp1) {
        // ============================ MMA warps ============================
        // one per tile, on different sub-partitions: while one waits for an
        // issue slot the other's products keep the tensor cores busy
        const int t = warp == kMmaWarp1 ? 1 : 0;
        if (lane == 0 && t < n_tiles) {
            int is = 0, ip = 0;  // next S and PV sub-stage of tile t
            const uint32_t t_s = taddr + t * kTileCols + kColS;
            const uint32_t t_q = taddr + t * kTileCols + kColQ;
            const uint32_t t_o = taddr + t * kTileCols + kColO;
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t spin = 0; ip < n_sub; ++spin) {
                // O_t += P_t(i) V^(i) once the softmax wrote P_t(i) and V^(i) is
                // written; the V^ buffer is free once every tile's PV(i) has
                // completed (one commit per tile); the epilogue waits for the last
                if (ip < is && mbar_test(&p_full[t], ip & 1) && mbar_test(&v_full[ip % kVBufs], (ip / kVBufs) & 1)) {
                    tc_fence_after();
                    const uint32_t aV = smem_u32(sV + (ip % kVBufs) * kKVBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_f16_ts(t_o, t_s + 8 * kk, desc_mn(aV, kk), kIdescPV, (ip > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&v_free[ip % kVBufs]);
                    if (ip == n_sub - 1) tc_commit(&o_free[t]);
                    ++ip;
                    continue;
                }
                // S_t(i) once K^(i) (and, the first time, Q_t) is written and
                // PV_t(i - 1), which reads P_t from the S_t columns, has been
                // issued: the tensor cores run one thread's MMAs in issue order,
                // so PV_t(i - 1) has read P_t before S_t(i) overwrites it, and the
                // commit that reports S_t(i) also reports PV_t(i - 1) complete
                // (the softmax may then rescale O_t); the K^ buffer is free once
                // every tile's S(i) has completed (one commit per tile)
                // turns: S_0(i) after S_1(i - 1) was issued, S_1(i) after S_0(i),
                // so one tile's softmax runs while the other's products do
                const bool turn = n_tiles < kTiles || (t == 0 ? sIssued[1] >= is : sIssued[0] > is);
                if (is < n_sub && ip == is && turn && mbar_test(&k_full[is & 1], (is >> 1) & 1) &&
                    (is > 0 || mbar_test(&q_full[t], 0))) {
                    tc_fence_after();
                    const uint32_t aKh = smem_u32(sK + (is & 1) * kKHalves * kKVBytes), aKl = aKh + kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc_mma_f16_ts(t_s, t_q + 8 * kk, desc_k(aKh, kSubKeys, kk), kIdescS, kk > 0);
                    if constexpr (KT == kKQ8_0) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            tc_mma_f16_ts(t_s, t_q + 8 * kk, desc_k(aKl, kSubKeys, kk), kIdescS, 1u);
                    }
                    tc_commit(&s_full[t]);
                    tc_commit(&k_free[is & 1]);
                    ++is;
                    sIssued[t] = is;
                    continue;
                }
                if ((spin & 255) == 255) {
                    if (*sAbort) { ok = false; break; }
                    if (globaltimer_ns() - t0 > kWaitLimitNs * 4) {
                        atomicOr(a.err, kErrWaitTimeout);
                        ok = false;
                        *sAbort = 1;
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp >= kSoftWarps) {
        // ============================ producer warps ============================
        const int pw = warp - kSoftWarps - (warp > kMmaWarp0);  // 0..4 (warps 8, 9, 11, 12, 13)
        const int ptid = pw * 32 + lane;
        for (int i = 0; i < n_sub; ++i) {
            const int r = i >> 1, sub = i & 1;
            const uint8_t* rb = raw + (r % kRS) * kRawBytes;
            if (sub == 0 && fail_wait(&raw_full[r % kRS], (r / kRS) & 1)) break;
            // the operand buffers hold the softmax warps' Q staging until every
            // tile's Q is in tensor memory
            if (i == 0 && (fail_wait(&q_full[0], 0) || (n_tiles > 1 && fail_wait(&q_full[1], 0)))) break;
            // ---- K^ hi / lo for keys [64 sub, 64 sub + 64) of the raw stage,
            //      once the S MMAs of sub-stage i - 2 released the buffer ----
            if (i >= 2 && fail_wait(&k_free[i & 1], ((i - 2) >> 1) & 1)) break;
            uint8_t* sKh = sK + (i & 1) * kKHalves * kKVBytes;
            uint8_t* sKl = sKh + kKVBytes;
            if constexpr (KT == kKF16) {
                // f16 K: K^ is the stored values; 16 B of raw row 2 key + dims/64
                // (swizzled by the TMA) to the operand tile's swizzled chunk
                for (int un = ptid; un < kSubKeys * 16; un += kProdThreads) {
                    const int kloc = un & 63, cc = un >> 6, hf = cc >> 3, c8 = cc & 7;
                    const int row = 2 * (sub * kSubKeys + kloc) + hf;
                    *reinterpret_cast<uint4*>(sKh + tile_off(kSubKeys, kloc, hf * 64 + 8 * c8)) =
                        *reinterpret_cast<const uint4*>(rb + kRawKq + row * 128 + ((c8 ^ (row & 7)) << 4));
                }
            } else {
            // each thread's (up to three) units: all shared-memory loads first,
            // so they are in flight together, then the conversions and stores
            constexpr int kKUnits = kSubKeys * 8, kKIters = (kKUnits + kProdThreads - 1) / kProdThreads;
            uint4 qk[kKIters];
            __half dk[kKIters];
#pragma unroll
            for (int it = 0; it < kKIters; ++it) {
                const int un = ptid + it * kProdThreads;
                if (un < kKUnits) {
                    const int kloc = un & 63, g = un >> 6, key = sub * kSubKeys + kloc;
                    qk[it] = *reinterpret_cast<const uint4*>(rb + kRawKq + key * 128 + ((g ^ (key & 7)) << 4));
                    dk[it] = *reinterpret_cast<const __half*>(rb + kRawKd + key * 8 + (g >> 1) * 2);
                }
            }
#pragma unroll
            for (int it = 0; it < kKIters; ++it) {
                const int un = ptid + it * kProdThreads;
                if (un >= kKUnits) break;
                const int kloc = un & 63, g = un >> 6;  // key in the sub-stage, 16-dim chunk
                const uint4 q = qk[it];
                const __half dh = dk[it];
                const __half2 d2 = __halves2half2(dh, dh);
                const __half2 bias = __float2half2_rn(1152.0f);
                const uint32_t w[4] = {q.x ^ 0x80808080u, q.y ^ 0x80808080u, q.z ^ 0x80808080u, q.w ^ 0x80808080u};
                uint32_t o[8], ol[8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    // bytes -> fp16 1024 + 128 + x (exact); minus 1152 -> x;
                    // hi = fp16(x d); lo = fp16(x d - hi) (the FMA forms x d - hi exactly)
                    const __half2 x01 = __hsub2(u2h(__byte_perm(w[u], 0x6464u, 0x5140u)), bias);
                    const __half2 x23 = __hsub2(u2h(__byte_perm(w[u], 0x6464u, 0x5342u)), bias);
                    const __half2 h01 = __hmul2(x01, d2), h23 = __hmul2(x23, d2);
                    o[2 * u] = h2u(h01);
                    o[2 * u + 1] = h2u(h23);
                    ol[2 * u] = h2u(__hfma2(x01, d2, __hneg2(h01)));
                    ol[2 * u + 1] = h2u(__hfma2(x23, d2, __hneg2(h23)));
                }
                const uint32_t off0 = tile_off(kSubKeys, kloc, g * 16), off1 = tile_off(kSubKeys, kloc, g * 16 + 8);
                *reinterpret_cast<uint4*>(sKh + off0) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(sKh + off1) = make_uint4(o[4], o[5], o[6], o[7]);
                *reinterpret_cast<uint4*>(sKl + off0) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                *reinterpret_cast<uint4*>(sKl + off1) = make_uint4(ol[4], ol[5], ol[6], ol[7]);
            }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&k_full[i & 1]);
            // ---- V^ [keys][dims], once the PV MMA of sub-stage i - 3 released
            //      the buffer; block b of a key: byte j = dims 32b+j (low), 32b+16+j (high) ----
            if (i >= kVBufs && fail_wait(&v_free[i % kVBufs], ((i - kVBufs) / kVBufs) & 1)) break;
            uint8_t* sVb = sV + (i % kVBufs) * kKVBytes;
            if constexpr (VT == kVQ8_0) {
                // Q8_0 V: V^ = fp16(d * q), the 32 codes of block blk of a key in
                // dims 32 blk .. 32 blk + 31 (exact int8 -> fp16, one rounding)
                for (int un = ptid; un < kSubKeys * kBlocks; un += kProdThreads) {
                    const int blk = un & 3, kloc = un >> 2;
                    const int key = sub * kSubKeys + kloc;
                    const uint4* src = reinterpret_cast<const uint4*>(rb + kRawVq + key * 128 + blk * 32);
                    const __half dh = *reinterpret_cast<const __half*>(rb + kRawVd + key * 8 + blk * 2);
                    const __half2 d2 = __halves2half2(dh, dh);
                    const __half2 bias = __float2half2_rn(1152.0f);
#pragma unroll
                    for (int hq = 0; hq < 2; ++hq) {
                        const uint4 q = src[hq];
                        const uint32_t w[4] = {q.x ^ 0x80808080u, q.y ^ 0x80808080u, q.z ^ 0x80808080u,
                                               q.w ^ 0x80808080u};
                        uint32_t o[8];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            o[2 * u] = h2u(__hmul2(__hsub2(u2h(__byte_perm(w[u], 0x6464u, 0x5140u)), bias), d2));
                            o[2 * u + 1] = h2u(__hmul2(__hsub2(u2h(__byte_perm(w[u], 0x6464u, 0x5342u)), bias), d2));
                        }
                        *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 32 * blk + 16 * hq)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 32 * blk + 16 * hq + 8)) =
                            make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
            } else if constexpr (VT == kVF16) {
                // F16 V: V^ is the stored values, copied 16 B (8 dims) at a time
                for (int un = ptid; un < kSubKeys * 16; un += kProdThreads) {
                    const int kloc = un >> 4, c = un & 15;
                    const int key = sub * kSubKeys + kloc;
                    *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 8 * c)) =
                        *reinterpret_cast<const uint4*>(rb + kRawVq + key * (kHeadDim * 2) + 16 * c);
                }
            } else
            {
            // each thread's (up to two) units: loads first, then conversions and stores
            constexpr int kVUnits = kSubKeys * kBlocks, kVIters = (kVUnits + kProdThreads - 1) / kProdThreads;
            uint4 qv[kVIters];
            __half dvv[kVIters], mvv[kVIters];
            uint32_t hvv[kVIters];
#pragma unroll
            for (int it = 0; it < kVIters; ++it) {
                const int un = ptid + it * kProdThreads;
                if (un < kVUnits) {
                    const int blk = un & 3, key = sub * kSubKeys + (un >> 2);
                    qv[it] = *reinterpret_cast<const uint4*>(rb + kRawVq + key * 64 + blk * 16);
                    dvv[it] = *reinterpret_cast<const __half*>(rb + kRawVd + key * 8 + blk * 2);
                    hvv[it] = 0;
                    if constexpr (v_has_fifth(VT)) hvv[it] = *reinterpret_cast<const uint32_t*>(rb + kRawVh + key * 16 + blk * 4);
                    if constexpr (v_has_min(VT)) mvv[it] = *reinterpret_cast<const __half*>(rb + kRawVm + key * 8 + blk * 2);
                }
            }
#pragma unroll
            for (int it = 0; it < kVIters; ++it) {
                const int un = ptid + it * kProdThreads;
                if (un >= kVUnits) break;
                // Q4_0 V: V^ = fp16(d * (q - 8)); Q5_0 V: the same nibbles with
                // the fifth bits added, V^ = fp16(d * (q - 16)); Q4_1 / Q5_1 V:
                // V^ = fp16(d * q + m) (one rounding)
                const int blk = un & 3, kloc = un >> 2;
                const uint4 q = qv[it];
                const __half dh = dvv[it];
                const uint32_t hw = hvv[it];
                const __half2 d2 = __halves2half2(dh, dh);
                __half2 m2 = __float2half2_rn(0.0f);
                if constexpr (v_has_min(VT)) m2 = __halves2half2(mvv[it], mvv[it]);
                const __half2 bias = __float2half2_rn(v_has_min(VT) ? 1024.0f : (VT == kVQ5_0 ? 1040.0f : 1032.0f));
                // code pair (exact in fp16) -> V^ pair
                auto val = [&](uint32_t bits) {
                    const __half2 x = __hsub2(u2h(bits | 0x64006400u), bias);
                    if constexpr (v_has_min(VT)) return h2u(__hfma2(x, d2, m2));
                    else return h2u(__hmul2(x, d2));
                };
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
                uint32_t lo[8], hi[8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t p01 = __byte_perm(w[u], 0u, 0x4140u);  // bytes 4u, 4u+1 at positions 0, 2
                    const uint32_t p23 = __byte_perm(w[u], 0u, 0x4342u);
                    lo[2 * u] = val((p01 & 0x000F000Fu) | fifth_bits(hw, 4 * u));
                    lo[2 * u + 1] = val((p23 & 0x000F000Fu) | fifth_bits(hw, 4 * u + 2));
                    hi[2 * u] = val(((p01 >> 4) & 0x000F000Fu) | fifth_bits(hw, 16 + 4 * u));
                    hi[2 * u + 1] = val(((p23 >> 4) & 0x000F000Fu) | fifth_bits(hw, 18 + 4 * u));
                }
                *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 32 * blk)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 32 * blk + 8)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
                *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 32 * blk + 16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sVb + tile_off(kSubKeys, kloc, 32 * blk + 24)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            }
            }
            // the stores above go to the tensor cores (async proxy); the raw
            // stage's reads are done before its buffer is handed back to TMA
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_cta(&v_full[i % kVBufs]);
                if (sub == 1) mbar_arrive_cta(&raw_free[r % kRS]);
            }
        }
    } else if (my_tile < n_tiles) {
        // ============================ softmax warps ============================
        {
            // Q tile into tensor memory: lane r = local query row (2 z + t) 128 + r
            // (rows past the head's rows are zero), dims 2c, 2c+1 in column Q + c.
            // The warp reads its 32 rows two at a time as whole 256-byte rows
            // (all sixteen loads in flight), transposes them through shared
            // memory (272-byte row stride: no bank conflicts either way) and each
            // thread stores its own row.  The staging area is the K^/V^ operand
            // buffers, which the producers write only after every tile's Q barrier.
            const int wrow0 = (2 * blockIdx.z + my_tile) * kMTile + (warp % kTileWarps) * 32;
            uint8_t* qst = sK + warp * (32 * 272);
            const int c16 = lane & 15;
            uint4 qa[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int lr = wrow0 + 2 * k + (lane >> 4);
                qa[k] = make_uint4(0, 0, 0, 0);
                if (lr < rows_head) {
                    const int j = lr / a.group, g = lr - j * a.group;
                    qa[k] = *reinterpret_cast<const uint4*>(a.q + ((size_t)j * a.n_qh + h * a.group + g) * kHeadDim +
                                                            c16 * 8);
                }
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
                *reinterpret_cast<uint4*>(qst + (2 * k + (lane >> 4)) * 272 + c16 * 16) = qa[k];
            __syncwarp();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t qv[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(qst + lane * 272 + (half * 8 + c) * 16);
                    qv[4 * c] = v.x; qv[4 * c + 1] = v.y; qv[4 * c + 2] = v.z; qv[4 * c + 3] = v.w;
                }
                tmem_st32u(taddr + lane_off + tcol + kColQ + half * 32, qv);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&q_full[my_tile]);
        }
        const int srow = (warp % kTileWarps) * 32 + lane;  // TMEM lane = query row of the tile
        const int lrow = (2 * blockIdx.z + my_tile) * kMTile + srow;
        const bool row_valid = lrow < rows_head;
        const bool warp_active = __any_sync(0xffffffffu, row_valid);
        const int qpos = row_valid ? a.pos0 + lrow / a.group : -1;
        const int kend = min(a.len - 1, qpos);  // last visible key position of this row
        const uint32_t t_s = taddr + tcol + kColS + lane_off, t_o = taddr + tcol + kColO + lane_off;
        float m_ref = -CUDART_INF_F, l_run = 0.0f;
        for (int i = 0; i < n_sub; ++i) {
            // S_t(i) is issued after PV_t(i - 1) and its commit covers both, so
            // once it has landed O_t is stable and the S_t columns may take P_t(i)
            const bool bad = fail_wait(&s_full[my_tile], i & 1);
            if (!__all_sync(0xffffffffu, !bad)) break;
            tc_fence_after();
            const int sg = raw0 + (i >> 1);
            const int kbase = (a.page0 + (sg >> 1)) * kPageTokens + (sg & 1) * kRawKeys + (i & 1) * kSubKeys;
            const bool tail = kbase + 63 > kend;  // keys past the row's causal end in this sub-stage
            if (warp_active) {
                uint32_t pk[32];
                float lsum = 0.0f, alpha = 1.0f;
                // p = 2^(s scale - m) with the reference max m, and the sub-stage's
                // sum; masked keys give 2^-inf = 0.  The scaling and the sums run
                // on packed pairs: the fewer instructions the softmax issues, the
                // sooner an MMA warp on the same sub-partition gets its turn.
                auto exp_row = [&](const float (&v)[64], float m) {
                    const float2 sc = make_float2(a.q_scale, a.q_scale), nm = make_float2(-m, -m);
                    float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);  // independent partial sums
#pragma unroll
                    for (int e = 0; e < 64; e += 4) {
                        const float2 x0 = fma2(make_float2(v[e], v[e + 1]), sc, nm);
                        const float2 x1 = fma2(make_float2(v[e + 2], v[e + 3]), sc, nm);
                        const float2 p01 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
                        const float2 p23 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
                        la = add2(la, p01);
                        lb = add2(lb, p23);
                        pk[e >> 1] = h2u(__floats2half2_rn(p01.x, p01.y));
                        pk[(e >> 1) + 1] = h2u(__floats2half2_rn(p23.x, p23.y));
                    }
                    const float2 l2 = add2(la, lb);
                    return l2.x + l2.y;
                };
                auto load_s = [&](float (&v)[64]) {
                    tmem_ld64(t_s, v);
                    if (tail) {
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (kbase + e > kend) v[e] = -CUDART_INF_F;
                    }
                };
                // Fast path: keep the reference max.  The sub-stage is accepted
                // when its sum is at most 2^8, so every p <= 2^8 as the lazy max
                // below guarantees; the row max is then never needed.
                bool slow = __any_sync(0xffffffffu, m_ref == -CUDART_INF_F);
                if (!slow) {
                    float v[64];
                    load_s(v);
                    lsum = exp_row(v, m_ref);
                    slow = __any_sync(0xffffffffu, !(lsum <= 256.0f));
                }
                if (slow) {
                    // the row max over the 64 keys (eight independent chains); the
                    // reference max moves only if it grew by more than 2^8
                    float v[64];
                    load_s(v);
                    float m8[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) m8[j] = v[j];
#pragma unroll
                    for (int e = 8; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], v[e]);
                    const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                           fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                    const float m_stage = mx * a.q_scale;
                    float m_use = m_ref;
                    if (m_stage > m_ref + 8.0f) m_use = m_stage;
                    const float mu = (m_use == -CUDART_INF_F) ? 0.0f : m_use;
                    alpha = (m_use == m_ref) ? 1.0f : ex2_approx(m_ref - mu);
                    m_ref = m_use;
                    lsum = exp_row(v, mu);
                }
                l_run = fmaf(l_run, alpha, lsum);
                tmem_st32u(t_s, pk);  // P_t over the first 32 S_t columns (waits for the store)
                // rescale the row of O_t (stable: S_t(i) landing means PV_t(i - 1) completed)
                if (i > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                    float o[32];
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        tmem_ld32(t_o + c * 32, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= alpha;
                        tmem_st32(t_o + c * 32, o);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&p_full[my_tile]);
        }
        // ---- epilogue: wait for the tile's last PV, write the split's partials ----
        const bool bad3 = (n_sub > 0) && fail_wait(&o_free[my_tile], 0);  // the tile's last PV
        tc_fence_after();
        if (__all_sync(0xffffffffu, !bad3 && ok) && warp_active) {
            const int split_g = a.split_base + blockIdx.x;
            const int j = lrow / a.group, g = lrow - j * a.group;
            const int grow = j * a.n_qh + h * a.group + g;
            // accumulate: fold in the record the previous launch left for this
            // (split, row): with M = max of the two reference maxima, O and l
            // are the 2^(m - M)-weighted sums (a record with l = 0 counts as empty)
            float w_new = 1.0f, w_old = 0.0f, m_out = m_ref, l_out = l_run;
            float2 prev = make_float2(-CUDART_INF_F, 0.0f);
            if (a.accumulate && row_valid) prev = a.part.ml[(size_t)split_g * a.n_rows + grow];
            if (prev.y > 0.0f) {
                if (l_run > 0.0f) {
                    m_out = fmaxf(prev.x, m_ref);
                    w_old = ex2_approx(prev.x - m_out);
                    w_new = ex2_approx(m_ref - m_out);
                } else {
                    m_out = prev.x;
                    w_old = 1.0f;
                    w_new = 0.0f;
                }
                l_out = w_old * prev.y + w_new * l_run;
            }
            // 32 columns of the warp's 32 rows at a time: each thread puts its
            // row's w_new-weighted O into shared memory (36-float row stride),
            // then 8 lanes take a row's 32 columns as 16-byte pieces, 4 rows per
            // instruction, so each row (and the previous record folded into
            // it) moves as one 128-byte line.  The staging area is the raw
            // stages: the tile's last PV has completed, so every raw stage has
            // landed and been dequantized.
            float* stg = reinterpret_cast<float*>(raw) + warp * (32 * 36);
            float* acc_split = a.part.acc + (size_t)split_g * a.n_rows * kHeadDim;
            const int sub_r = lane >> 3, q4 = lane & 7;  // row within a group of 4, 16-byte piece of the row
            float wo_k[8];
            int gr_k[8];  // record row of row 4 k + sub_r, -1 when the row is past the head's rows
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                wo_k[k] = __shfl_sync(0xffffffffu, w_old, 4 * k + sub_r);
                gr_k[k] = __shfl_sync(0xffffffffu, row_valid ? grow : -1, 4 * k + sub_r);
            }
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float o[32];
                tmem_ld32(t_o + c * 32, o);
                const float wn = (n_sub == 0) ? 0.0f : w_new;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(stg + lane * 36 + 4 * j) =
                        make_float4(o[4 * j] * wn, o[4 * j + 1] * wn, o[4 * j + 2] * wn, o[4 * j + 3] * wn);
                __syncwarp();
                float4 pv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    pv[k] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (wo_k[k] != 0.0f)
                        pv[k] = *reinterpret_cast<const float4*>(acc_split + (size_t)gr_k[k] * kHeadDim + c * 32 + 4 * q4);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (gr_k[k] < 0) continue;
                    const float4 sv = *reinterpret_cast<const float4*>(stg + (4 * k + sub_r) * 36 + 4 * q4);
                    const float wo = wo_k[k];
                    *reinterpret_cast<float4*>(acc_split + (size_t)gr_k[k] * kHeadDim + c * 32 + 4 * q4) =
                        make_float4(fmaf(wo, pv[k].x, sv.x), fmaf(wo, pv[k].y, sv.y), fmaf(wo, pv[k].z, sv.z),
                                    fmaf(wo, pv[k].w, sv.w));
                }
                __syncwarp();
            }
            if (row_valid) a.part.ml[(size_t)split_g * a.n_rows + grow] = make_float2(m_out, l_out);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(taddr, kTmemCols);
    }
}

template <int VT, int KT = kKQ8_0, bool ZC = false>
static cudaError_t launch_chunk_t(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits, cudaStream_t s) {
    // devices whose shared-memory opt-in is done (calls from several host
    // threads may race to set a bit; the attribute call is idempotent)
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !(configured.load(std::memory_order_acquire) & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(chunk_mma_kernel<VT, KT, ZC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)TcGeom<VT, KT>::kSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
    }
    const int m_tiles = (a.n_q * a.group + kMTile - 1) / kMTile;
    dim3 grid(n_splits, a.n_kv, (m_tiles + kTiles - 1) / kTiles);
    chunk_mma_kernel<VT, KT, ZC><<<grid, kTcThreads, TcGeom<VT, KT>::kSmem, s>>>(a, *kmap);
    return cudaGetLastError();
}

}  // namespace

template <bool ZC>
static cudaError_t launch_chunk_types(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits, cudaStream_t s) {
    if (a.k_type == kKF16) return launch_chunk_t<kVF16, kKF16, ZC>(a, kmap, n_splits, s);
    switch (a.v_type) {
        case kVQ8_0: return launch_chunk_t<kVQ8_0, kKQ8_0, ZC>(a, kmap, n_splits, s);
        case kVQ5_0: return launch_chunk_t<kVQ5_0, kKQ8_0, ZC>(a, kmap, n_splits, s);
        case kVQ4_1: return launch_chunk_t<kVQ4_1, kKQ8_0, ZC>(a, kmap, n_splits, s);
        case kVQ5_1: return launch_chunk_t<kVQ5_1, kKQ8_0, ZC>(a, kmap, n_splits, s);
        case kVF16: return launch_chunk_t<kVF16, kKQ8_0, ZC>(a, kmap, n_splits, s);
        default: return launch_chunk_t<kVQ4_0, kKQ8_0, ZC>(a, kmap, n_splits, s);
    }
}

cudaError_t launch_chunk_mma(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits, cudaStream_t s) {
    return launch_chunk_types<false>(a, kmap, n_splits, s);
}

cudaError_t launch_chunk_mma_zero_copy(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits, cudaStream_t s) {
    return launch_chunk_types<true>(a, kmap, n_splits, s);
}

}  // namespace kvs

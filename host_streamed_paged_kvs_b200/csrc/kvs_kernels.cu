// kvs_kernels.cu -- sm_100a kernels of the streamed quantized-KV attention path:
//   K1 append_kernel  : fp16 K/V rows -> Q8_0 K / Q4_0 V blocks, written to the
//                       pinned host history (mapped) and to the resident slot;
//   K2 decode_kernel  : split-K flash-decode over resident pages or ring slots,
//                       K/V dequantized in registers, per-split (m, l, acc);
//   K3 merge_kernel   : log-sum-exp merge of the split partials.
//
// Method sources: "RaymondHuang210129/llama.cpp-adaptive-kv-streaming" (Summary:
// pinned authoritative history, resident pages + one shared ring, Q8_0 K /
// Q4_0 V) and "Feature/adaptive kv stream integration" (PR #326, section 1:
// attention with streaming is the same computation as without it).
#include <cuda_fp16.h>
#include <math_constants.h>

#include <algorithm>

#include <atomic>

#include "kvs_internal.h"
#include "kvs_ptx.cuh"

namespace kvs {

// int8 byte i of w -> exact float, via 2^23 + (b + 128) - (2^23 + 128)
__device__ __forceinline__ float s8_to_f(uint32_t w_biased, int i) {
    return __uint_as_float(__byte_perm(w_biased, 0x4B00u, 0x5440u + i)) - 8388736.0f;
}
// 4-bit code c -> exact float (c - 8)
__device__ __forceinline__ float q4_to_f(uint32_t c) {
    return __uint_as_float(0x4B000000u | c) - 8388616.0f;
}

// ----------------------------------------------------------------------------
// K1: quantize-on-append.  One warp per (token, kv head) row of 128 values;
// lane l owns dims 4l..4l+3, so 8 lanes form one 32-value block.
// Q8_0: d = amax/127 (binary32, correctly rounded), q = roundf(x/d).
// Q4_0: m = value of largest |x| (first index on ties), d = m/-8,
//       q = min(15, trunc(x/d + 8.5)), d == 0 -> q = 8.
// Q5_0: the same with 32 levels: d = m/-16, q = min(31, trunc(x/d + 16.5)),
//       d == 0 -> q = 16; the low 4 bits are packed as Q4_0's codes, the
//       fifth bits in one 32-bit word per block (bit j = code j).
// Q4_1 / Q5_1: lo, hi = block minimum and maximum (first index on ties),
//       d = (hi - lo)/L with L = 15 / 31, q = min(L, trunc((x - lo)/d + 0.5)),
//       d == 0 -> q = 0; the block minimum is stored as an fp16 m.
// The stored scales are the fp16 (round-to-nearest-even) values of d.
// K is always Q8_0; V is F16 (VT = 1, the values as they are), Q4_0 (2),
// Q4_1 (3), Q5_0 (6), Q5_1 (7) or Q8_0 (8).
// ----------------------------------------------------------------------------
// Q8_0 of the 32-value block spread over 8 lanes (4 values each): the lane's
// 4 codes packed in one word (byte u = code of value u), and the block scale
__device__ __forceinline__ uint32_t q8_0_lane(const float (&x)[4], float& d) {
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    d = __fdiv_rn(amax, 127.0f);
    uint32_t w = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int q = 0;
        if (d != 0.0f) q = static_cast<int>(roundf(__fdiv_rn(x[u], d)));
        w |= (static_cast<uint32_t>(q) & 0xffu) << (8 * u);
    }
    return w;
}

template <int VT, int KT = kKQ8_0>
__global__ void __launch_bounds__(128) append_kernel(const AppendArgs a) {
    using G = PageGeom<VT, KT>;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= a.n_tok * a.n_kv) return;
    const int tok = row / a.n_kv;
    const int h = row - tok * a.n_kv;
    const int pos = a.pos0 + tok;
    const int page = pos >> 8;
    const int t = pos & 255;
    const int b = lane >> 3;  // block of this lane
    const int i = lane & 7;   // position of the lane in its block

    const uint2 kraw = *reinterpret_cast<const uint2*>(a.k + (size_t)row * kHeadDim + 4 * lane);
    const uint2 vraw = *reinterpret_cast<const uint2*>(a.v + (size_t)row * kHeadDim + 4 * lane);
    float xk[4], xv[4];
    {
        const __half2 k01 = *reinterpret_cast<const __half2*>(&kraw.x);
        const __half2 k23 = *reinterpret_cast<const __half2*>(&kraw.y);
        const __half2 v01 = *reinterpret_cast<const __half2*>(&vraw.x);
        const __half2 v23 = *reinterpret_cast<const __half2*>(&vraw.y);
        xk[0] = __low2float(k01); xk[1] = __high2float(k01);
        xk[2] = __low2float(k23); xk[3] = __high2float(k23);
        xv[0] = __low2float(v01); xv[1] = __high2float(v01);
        xv[2] = __low2float(v23); xv[3] = __high2float(v23);
    }

    // ---- Q8_0 (K) ----
    float dk;
    const uint32_t kq = q8_0_lane(xk, dk);
    const __half dk_h = __float2half_rn(dk);

    if constexpr (VT == kVQ8_0) {
        // ---- Q8_0 (V) ----
        float dv;
        const uint32_t vq = q8_0_lane(xv, dv);
        const __half dv_h = __float2half_rn(dv);
        auto store = [&](uint8_t* ph) {
            *reinterpret_cast<uint32_t*>(ph + kOffKq + t * kHeadDim + 4 * lane) = kq;
            *reinterpret_cast<uint32_t*>(ph + G::kOffVq + t * kHeadDim + 4 * lane) = vq;
            if (i == 0) {
                *reinterpret_cast<__half*>(ph + kOffKd + t * 8 + 2 * b) = dk_h;
                *reinterpret_cast<__half*>(ph + G::kOffVd + t * 8 + 2 * b) = dv_h;
            }
        };
        store(a.host_layer + (size_t)page * a.page_bytes + (size_t)h * G::kHeadBytes);
        if (page >= a.first_resident_page) {
            const int slot = page % a.n_resident;
            store(a.res_layer + (size_t)slot * a.page_bytes + (size_t)h * G::kHeadBytes);
        }
        return;
    }

    if constexpr (VT == kVF16) {
        // ---- F16 (V): the values as they are; F16 K (the f16-f16 pair) likewise ----
        auto store = [&](uint8_t* ph) {
            if constexpr (KT == kKF16) {
                *reinterpret_cast<uint2*>(ph + G::kOffKq + t * G::kKqRow + 8 * lane) = kraw;
            } else {
                *reinterpret_cast<uint32_t*>(ph + kOffKq + t * kHeadDim + 4 * lane) = kq;
                if (i == 0) *reinterpret_cast<__half*>(ph + kOffKd + t * 8 + 2 * b) = dk_h;
            }
            *reinterpret_cast<uint2*>(ph + G::kOffVq + t * G::kVqRow + 8 * lane) = vraw;
        };
        store(a.host_layer + (size_t)page * a.page_bytes + (size_t)h * G::kHeadBytes);
        if (page >= a.first_resident_page) {
            const int slot = page % a.n_resident;
            store(a.res_layer + (size_t)slot * a.page_bytes + (size_t)h * G::kHeadBytes);
        }
        return;
    }

    if constexpr (v_has_min(VT)) {
        // ---- Q4_1 / Q5_1 (V): block minimum and maximum, first index on ties ----
        float lo = xv[0], hi = xv[0];
        int ilo = 4 * i, ihi = 4 * i;
#pragma unroll
        for (int u = 1; u < 4; ++u) {
            if (xv[u] < lo) { lo = xv[u]; ilo = 4 * i + u; }
            if (xv[u] > hi) { hi = xv[u]; ihi = 4 * i + u; }
        }
#pragma unroll
        for (int off = 1; off <= 4; off <<= 1) {
            const float plo = __shfl_xor_sync(0xffffffffu, lo, off);
            const int pilo = __shfl_xor_sync(0xffffffffu, ilo, off);
            const float phi = __shfl_xor_sync(0xffffffffu, hi, off);
            const int pihi = __shfl_xor_sync(0xffffffffu, ihi, off);
            if (plo < lo || (plo == lo && pilo < ilo)) { lo = plo; ilo = pilo; }
            if (phi > hi || (phi == hi && pihi < ihi)) { hi = phi; ihi = pihi; }
        }
        constexpr int kL = G::kLevels;
        const float dv = __fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(kL));
        uint32_t codes = 0, high = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            int q = 0;
            if (dv != 0.0f) q = min(kL, static_cast<int>(__fadd_rn(__fdiv_rn(__fsub_rn(xv[u], lo), dv), 0.5f)));
            codes |= static_cast<uint32_t>(q & 15) << (8 * u);
            high |= static_cast<uint32_t>(q >> 4) << (4 * i + u);
        }
        const uint32_t partner = __shfl_xor_sync(0xffffffffu, codes, 4);
        const uint32_t vq = codes | (partner << 4);
        if constexpr (v_has_fifth(VT)) {
            high |= __shfl_xor_sync(0xffffffffu, high, 1);
            high |= __shfl_xor_sync(0xffffffffu, high, 2);
            high |= __shfl_xor_sync(0xffffffffu, high, 4);
        }
        const __half dv_h = __float2half_rn(dv), mv_h = __float2half_rn(lo);
        auto store = [&](uint8_t* ph) {
            *reinterpret_cast<uint32_t*>(ph + kOffKq + t * kHeadDim + 4 * lane) = kq;
            if (i == 0) {
                *reinterpret_cast<__half*>(ph + kOffKd + t * 8 + 2 * b) = dk_h;
                *reinterpret_cast<__half*>(ph + G::kOffVd + t * 8 + 2 * b) = dv_h;
                *reinterpret_cast<__half*>(ph + G::kOffVm + t * 8 + 2 * b) = mv_h;
                if constexpr (v_has_fifth(VT)) *reinterpret_cast<uint32_t*>(ph + G::kOffVh + t * 16 + 4 * b) = high;
            }
            if (i < 4) *reinterpret_cast<uint32_t*>(ph + G::kOffVq + t * 64 + b * 16 + 4 * i) = vq;
        };
        store(a.host_layer + (size_t)page * a.page_bytes + (size_t)h * G::kHeadBytes);
        if (page >= a.first_resident_page) {
            const int slot = page % a.n_resident;
            store(a.res_layer + (size_t)slot * a.page_bytes + (size_t)h * G::kHeadBytes);
        }
        return;
    }

    // ---- Q4_0 / Q5_0 (V) ----
    constexpr bool kQ5 = VT == kVQ5_0;
    constexpr float kNegLevels = kQ5 ? -16.0f : -8.0f;
    constexpr float kRoundOff = kQ5 ? 16.5f : 8.5f;
    constexpr int kTop = kQ5 ? 31 : 15, kMid = kQ5 ? 16 : 8;
    float va = 0.0f, vm = 0.0f;
    int vi = 1 << 30;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const float ax = fabsf(xv[u]);
        if (ax > va) { va = ax; vm = xv[u]; vi = 4 * i + u; }
    }
#pragma unroll
    for (int off = 1; off <= 4; off <<= 1) {
        const float pa = __shfl_xor_sync(0xffffffffu, va, off);
        const float pm = __shfl_xor_sync(0xffffffffu, vm, off);
        const int pi = __shfl_xor_sync(0xffffffffu, vi, off);
        if (pa > va || (pa == va && pi < vi)) { va = pa; vm = pm; vi = pi; }
    }
    const float dv = __fdiv_rn(vm, kNegLevels);
    uint32_t codes = 0;  // 4 codes of this lane, one per byte
    uint32_t high = 0;   // Q5_0: bit 4 of code 4i+u at bit 4i+u
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int q = kMid;
        if (dv != 0.0f) q = min(kTop, static_cast<int>(__fadd_rn(__fdiv_rn(xv[u], dv), kRoundOff)));
        codes |= static_cast<uint32_t>(q & 15) << (8 * u);
        high |= static_cast<uint32_t>(q >> 4) << (4 * i + u);
    }
    const uint32_t partner = __shfl_xor_sync(0xffffffffu, codes, 4);  // codes j+16 for lanes i<4
    const uint32_t vq = codes | (partner << 4);  // byte u: q_(4i+u) | q_(4i+u+16) << 4 (low 4 bits)
    if constexpr (kQ5) {
        high |= __shfl_xor_sync(0xffffffffu, high, 1);
        high |= __shfl_xor_sync(0xffffffffu, high, 2);
        high |= __shfl_xor_sync(0xffffffffu, high, 4);
    }
    const __half dv_h = __float2half_rn(dv);

    // ---- stores: host history (always) and resident slot (if resident) ----
    auto store = [&](uint8_t* ph) {
        *reinterpret_cast<uint32_t*>(ph + kOffKq + t * kHeadDim + 4 * lane) = kq;
        if (i == 0) {
            *reinterpret_cast<__half*>(ph + kOffKd + t * 8 + 2 * b) = dk_h;
            *reinterpret_cast<__half*>(ph + G::kOffVd + t * 8 + 2 * b) = dv_h;
            if constexpr (kQ5) *reinterpret_cast<uint32_t*>(ph + G::kOffVh + t * 16 + 4 * b) = high;
        }
        if (i < 4) *reinterpret_cast<uint32_t*>(ph + G::kOffVq + t * 64 + b * 16 + 4 * i) = vq;
    };
    store(a.host_layer + (size_t)page * a.page_bytes + (size_t)h * G::kHeadBytes);
    if (page >= a.first_resident_page) {
        const int slot = page % a.n_resident;
        store(a.res_layer + (size_t)slot * a.page_bytes + (size_t)h * G::kHeadBytes);
    }
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
    const int rows = a.n_tok * a.n_kv;
    if (a.k_type == kKF16)
        append_kernel<kVF16, kKF16><<<(rows + 3) / 4, 128, 0, s>>>(a);
    else if (a.v_type == kVQ8_0)
        append_kernel<kVQ8_0><<<(rows + 3) / 4, 128, 0, s>>>(a);
    else if (a.v_type == kVQ5_0)
        append_kernel<kVQ5_0><<<(rows + 3) / 4, 128, 0, s>>>(a);
    else if (a.v_type == kVQ4_1)
        append_kernel<kVQ4_1><<<(rows + 3) / 4, 128, 0, s>>>(a);
    else if (a.v_type == kVQ5_1)
        append_kernel<kVQ5_1><<<(rows + 3) / 4, 128, 0, s>>>(a);
    else if (a.v_type == kVF16)
        append_kernel<kVF16><<<(rows + 3) / 4, 128, 0, s>>>(a);
    else
        append_kernel<kVQ4_0><<<(rows + 3) / 4, 128, 0, s>>>(a);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// K2: split-K flash-decode.  CTA = (split, kv head, row group), 256 threads.
// The pages of one launch are consumed as 128-token half-page stages; a split
// is an equal share of consecutive stages (the launch's n_splits splits).
// Stage bytes land in shared memory through TMA: the K quants with the
// 128-byte swizzle (a thread reading its key's row then hits distinct banks
// while the query chunk it multiplies is a broadcast), the K scales, V codes
// and V scales as 1-D bulk copies; three stages are in flight.  Every warp
// owns 16 keys of each stage end to end, with its own online-softmax state,
// and does its math on the tensor cores with warp-level mma.sync m16n8k16
// (fp16 operands, fp32 accumulate; the <= 8 query rows of a row group fill
// rows 0..7 of the 16-row tile):
//   QK^T : int8 K codes are exact in fp16; per 32-dim block the MMA gives the
//          block's partial score in fp32 and the block's K scale multiplies it;
//   softmax: warp-local lazy running max per row (log2 domain);
//   PV   : the probability times the V scale of each (key, block) is the A
//          operand (one fp16 rounding), the V codes (q - 8 for Q4_0, q - 16
//          for Q5_0, q for Q8_0) exact in fp16 are the B operand; for Q4_1 /
//          Q5_1 the A operand is p and B the value fp16(q d + m), for F16 V
//          p and the stored value.
// A stage buffer is refilled once all eight warps have released it (an
// mbarrier with eight arrivals); there is no CTA-wide barrier in the loop.  At
// the end the eight warps' (m, l, O) are merged into the split's partial.
// ----------------------------------------------------------------------------
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStageKeys = 128;
constexpr int kWarpKeys = kStageKeys / kWarps;                    // 16
constexpr int kStageKq = 0;
constexpr int kStageKd = kStageKeys * kHeadDim;                  // 16384
constexpr int kStageVq = kStageKd + kStageKeys * kBlocks * 2;      // 17408
constexpr int kStageVd = kStageVq + kStageKeys * kHeadDim / 2;     // 25600
constexpr int kStageBytes = kStageVd + kStageKeys * kBlocks * 2;   // 26624
constexpr int kStages = 3;
constexpr int kMaxRows = 8;
constexpr int kQFragBytes = 32 * 16 * 4;    // Q operand fragments: 16 words per lane
constexpr size_t kOffQ = kStages * kStageBytes;
constexpr size_t kOffKend = kOffQ + kQFragBytes;                                 // sQf
constexpr size_t kOffBar = kOffKend + kMaxRows * 4;                              // sKend
constexpr size_t kDecodeSmem = 1024 /*align slack*/ + kOffBar + 2 * kStages * 8;
static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-B swizzle alignment");
static_assert(kWarps * kMaxRows * (kHeadDim + 2) * 4 <= kStages * kStageBytes, "merge scratch fits");

// Stage and shared-memory geometry by V type: a Q8_0-V stage carries 128 B of
// V codes per key (34,816 B per stage) and an F16-V stage 256 B of values
// (50,176 B), so they keep two stages in flight to stay at two CTAs per SM;
// a Q5_0-V stage adds 16 B of fifth bits per key (28,672 B) and keeps three.
// An f16-f16 stage carries 256 B of K values and 256 B of V values per key
// (65,536 B): two stages, one CTA per SM.
template <int VT, int KT = kKQ8_0>
struct DecGeom {
    using PG = PageGeom<VT, KT>;
    static constexpr int kVqRow = PG::kVqRow;
    static constexpr int kVhRow = PG::kVhRow;
    static constexpr int kVmRow = PG::kVmRow;
    static constexpr int kKRows = kStageKeys * PG::kKqRow / 128;          // 128-byte K rows per stage
    static constexpr int kStageKd = kStageKeys * PG::kKqRow;               // 16384 for Q8_0 K
    static constexpr int kStageVq = kStageKd + kStageKeys * PG::kKdRow;   // 17408 for Q8_0 K
    static constexpr int kStageVh = kStageVq + kStageKeys * kVqRow;
    static constexpr int kStageVd = kStageVh + kStageKeys * kVhRow;
    static constexpr int kStageVm = kStageVd + kStageKeys * PG::kVdRow;
    static constexpr int kStageBytes = kStageVm + kStageKeys * kVmRow;
    static constexpr int kStages = (VT == kVQ8_0 || VT == kVF16) ? 2 : 3;
    static constexpr size_t kOffQ = (size_t)kStages * kStageBytes;
    static constexpr size_t kOffKend = kOffQ + kQFragBytes;
    static constexpr size_t kOffBar = kOffKend + kMaxRows * 4;
    static constexpr size_t kSmem = 1024 + kOffBar + 2 * kStages * 8;
    static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-B swizzle alignment");
    static_assert(kWarps * kMaxRows * (kHeadDim + 2) * 4 <= kStages * kStageBytes, "merge scratch fits");
};
static_assert(DecGeom<kVQ4_0>::kStageBytes == kStageBytes && DecGeom<kVQ4_0>::kSmem == kDecodeSmem,
              "Q4_0 decode geometry");
static_assert(2 * DecGeom<kVQ8_0>::kSmem <= 232448, "two Q8_0-V CTAs per SM");
static_assert(2 * DecGeom<kVQ5_0>::kSmem <= 232448 && DecGeom<kVQ5_0>::kStageBytes == 28672,
              "two Q5_0-V CTAs per SM");
static_assert(2 * DecGeom<kVQ4_1>::kSmem <= 232448 && DecGeom<kVQ4_1>::kStageBytes == 27648,
              "two Q4_1-V CTAs per SM");
static_assert(2 * DecGeom<kVQ5_1>::kSmem <= 232448 && DecGeom<kVQ5_1>::kStageBytes == 29696,
              "two Q5_1-V CTAs per SM");
static_assert(2 * DecGeom<kVF16>::kSmem <= 232448 && DecGeom<kVF16>::kStageBytes == 50176,
              "two F16-V CTAs per SM");
static_assert(DecGeom<kVF16, kKF16>::kSmem <= 232448 && DecGeom<kVF16, kKF16>::kStageBytes == 65536,
              "one f16-f16 CTA per SM");

size_t decode_smem_bytes() { return kDecodeSmem; }

// 2^x with the hardware approximation (flush-to-zero; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// D += A B, m16n8k16, fp16 operands, fp32 accumulate; the A rows 8..15 are
// zero (a1 = a3 = 0): a0 = {row g, k 2q..2q+1}, a2 = {row g, k 2q+8..2q+9}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2u(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}


// ZC = true: the pages are read in place from mapped pinned host memory (the
// history) by warp 0's 16-byte asynchronous copies instead of TMA, one stage
// = 1664 copies, 52 per lane, the K quants placed in the same 128-byte
// swizzle the tensor map produces
template <int ROWS, bool ZC, int VT, int KT>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap) {
    using G = DecGeom<VT, KT>;
    using PG = PageGeom<VT, KT>;
    constexpr int kStages = G::kStages;
    constexpr int kStageBytes = G::kStageBytes;
    constexpr int kStageKd = G::kStageKd;
    constexpr int kStageVq = G::kStageVq;
    constexpr int kStageVh = G::kStageVh;
    constexpr int kStageVd = G::kStageVd;
    constexpr int kStageVm = G::kStageVm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* stage = smem;
    uint32_t* sQf = reinterpret_cast<uint32_t*>(smem + G::kOffQ);  // [4 blocks][32 lanes][4] Q fragments
    int* sKend = reinterpret_cast<int*>(smem + G::kOffKend);           // last visible key per row
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::kOffBar);   // [kStages]
    uint64_t* empty = full + kStages;                               // [kStages]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    const int row_begin = blockIdx.z * ROWS;
    const int rows_here = min(ROWS, a.n_q * a.group - row_begin);
    const int n_stages_all = 2 * a.n_units;
    const int st0 = (int)(((long)blockIdx.x * n_stages_all) / a.n_splits);
    const int n_st = (int)(((long)(blockIdx.x + 1) * n_stages_all) / a.n_splits) - st0;

    // Q as the tensor-core A operand, one 16-word fragment set per lane
    // (the same for every warp): lane (g, q) holds, for k-step kk = 2b + s,
    // row g's fp16 dims {d0, d0+1} and {d0+2, d0+3}, d0 = 32b + 8q + 4s
    // (zero for rows past the CTA's rows)
    if (tid < 32) {
        const int g = tid >> 2, q = tid & 3;
        const bool vr = g < rows_here;
        const int lr = row_begin + g;
        const __half* qrow = a.q + ((size_t)(lr / a.group) * a.n_qh + h * a.group + (lr % a.group)) * kHeadDim;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int d0 = 32 * (kk >> 1) + 8 * q + 4 * (kk & 1);
            const uint2 v = vr ? *reinterpret_cast<const uint2*>(qrow + d0) : make_uint2(0u, 0u);
            uint32_t* qf = sQf + ((kk >> 1) * 32 + tid) * 4 + 2 * (kk & 1);  // lane-contiguous per block
            qf[0] = v.x;
            qf[1] = v.y;
        }
    }
    if (tid < ROWS)  // row r sees keys 0 .. min(len-1, its query position); padding rows none
        sKend[tid] = (tid < rows_here) ? min(a.len - 1, a.pos0 + (row_begin + tid) / a.group) : -1;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], ZC ? 32 : 1);
            mbar_init(&empty[s], kWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](int i) {  // i: stage index within this split
        const int sg = st0 + i;
        const int u = sg >> 1, half = sg & 1;
        const int slot = (a.slot0 + u) % a.region_slots;
        const uint8_t* ph = a.region + ((size_t)slot * a.n_kv + h) * PG::kHeadBytes;
        uint8_t* dst = stage + (i % kStages) * kStageBytes;
        uint64_t* b = &full[i % kStages];
        if constexpr (ZC) {
            // K quants (or f16 K values): 128-byte row r of the half page,
            // 16-byte chunk k -> swizzled
            const uint8_t* kq = ph + PG::kOffKq + half * (kStageKeys * PG::kKqRow);
#pragma unroll 4
            for (int c = lane; c < G::kKRows * 8; c += 32) {
                const int r = c >> 3, k = c & 7;
                cp_async16(dst + kStageKq + r * 128 + ((k ^ (r & 7)) << 4), kq + r * 128 + k * 16);
            }
            const uint8_t* kd = ph + PG::kOffKd + half * (kStageKeys * PG::kKdRow);
            const uint8_t* vq = ph + PG::kOffVq + half * (kStageKeys * PG::kVqRow);
            const uint8_t* vd = ph + PG::kOffVd + half * (kStageKeys * kBlocks * 2);
            for (int c = lane; c < kStageKeys * kBlocks * 2 / 16; c += 32) {
                if constexpr (PG::kKdRow > 0) cp_async16(dst + kStageKd + c * 16, kd + c * 16);
                if constexpr (PG::kVdRow > 0) cp_async16(dst + kStageVd + c * 16, vd + c * 16);
            }
#pragma unroll 4
            for (int c = lane; c < kStageKeys * PG::kVqRow / 16; c += 32)
                cp_async16(dst + kStageVq + c * 16, vq + c * 16);
            if constexpr (PG::kVhRow > 0) {
                const uint8_t* vh = ph + PG::kOffVh + half * (kStageKeys * PG::kVhRow);
                for (int c = lane; c < kStageKeys * PG::kVhRow / 16; c += 32)
                    cp_async16(dst + kStageVh + c * 16, vh + c * 16);
            }
            if constexpr (PG::kVmRow > 0) {
                const uint8_t* vm = ph + PG::kOffVm + half * (kStageKeys * PG::kVmRow);
                for (int c = lane; c < kStageKeys * PG::kVmRow / 16; c += 32)
                    cp_async16(dst + kStageVm + c * 16, vm + c * 16);
            }
            cp_async_arrive(b);
        } else {
            mbar_expect_tx(b, kStageBytes);
            const int krow = ((a.region_slot_base + slot) * a.n_kv + h) * PG::kRows + half * G::kKRows;
#pragma unroll
            for (int kr = 0; kr < G::kKRows; kr += 128)  // boxes of 128 rows of 128 B
                tma_load_2d(dst + kStageKq + kr * 128, &kmap, 0, krow + kr, b);
            if constexpr (PG::kKdRow > 0)
                bulk_load(dst + kStageKd, ph + PG::kOffKd + half * (kStageKeys * PG::kKdRow), kStageKeys * PG::kKdRow, b);
            bulk_load(dst + kStageVq, ph + PG::kOffVq + half * (kStageKeys * PG::kVqRow), kStageKeys * PG::kVqRow, b);
            if constexpr (PG::kVhRow > 0)
                bulk_load(dst + kStageVh, ph + PG::kOffVh + half * (kStageKeys * PG::kVhRow), kStageKeys * PG::kVhRow, b);
            if constexpr (PG::kVdRow > 0)
                bulk_load(dst + kStageVd, ph + PG::kOffVd + half * (kStageKeys * kBlocks * 2), kStageKeys * kBlocks * 2, b);
            if constexpr (PG::kVmRow > 0)
                bulk_load(dst + kStageVm, ph + PG::kOffVm + half * (kStageKeys * PG::kVmRow), kStageKeys * PG::kVmRow, b);
        }
    };
    // the producer: thread 0 (TMA), or all of warp 0 (zero-copy)
    const bool producer = ZC ? (warp == 0) : (tid == 0);
    int next_issue = 0;
    if (producer) {
        for (; next_issue < kStages && next_issue < n_st; ++next_issue) issue(next_issue);
    }

    // ---- tensor-core math (mma.sync m16n8k16: fp16 operands, fp32 accumulate) ----
    // Row g = lane / 4 of the MMA tile is query row g of this CTA (rows past
    // rows_here, and the tile's rows 8..15, are zero); q = lane % 4.
    // QK^T, per 32-dim block b: two k-steps s; MMA k-index 2q+{0,1} and
    //   2q+8+{0,1} of k-step s stand for dims 32b+8q+4s+{0,1} and {2,3}, so a
    //   lane's K operand is 4 consecutive int8 of its key's row (exact in fp16)
    //   and the block's scale multiplies the block's fp32 partial score.
    // PV: n-tile nt = 4b + m holds dims 32b + 4n + m (column n); the MMA
    //   k-index runs over the warp's 16 keys in the order of the score tile's
    //   columns, and the probabilities carry the V scale of block b (one fp16
    //   rounding of p * d_v; the codes q - 8 are exact in fp16).
    const int g = lane >> 2, q = lane & 3;
    const uint4* qfrag = reinterpret_cast<const uint4*>(sQf) + lane;  // block b: qfrag[32 b]
    const int kend = g < ROWS ? sKend[g] : -1;  // last visible key of this lane's row
    float o[16][2];                              // O (row g; dims of n-tile nt, columns 2q, 2q+1)
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = 0.0f;
    float zr0 = 0.0f, zr1 = 0.0f;  // the tile's rows 8..15: zero operands keep them zero
    float m_run = -CUDART_INF_F, l_run = 0.0f;
    bool ok = true;
    const __half2 b1152 = __float2half2_rn(1152.0f), b1032 = __float2half2_rn(1032.0f);
    const __half2 b1040 = __float2half2_rn(1040.0f), b1024 = __float2half2_rn(1024.0f);

    for (int i = 0; i < n_st; ++i) {
        // producer: keep the next two stages in flight (it waits for all
        // warps to release the buffer it refills)
        if (producer) {
            for (; next_issue < n_st && next_issue < i + kStages; ++next_issue) {
                const int prev = next_issue - kStages;  // last stage that used this buffer
                if (prev >= 0 && !mbar_wait_bounded(&empty[prev % kStages], (prev / kStages) & 1, a.err)) {
                    ok = false;
                    break;
                }
                issue(next_issue);
            }
        }
        const uint8_t* sb = stage + (i % kStages) * kStageBytes;
        if (!mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1, a.err)) ok = false;
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        const int sg = st0 + i;
        const int kbase = (a.page0 + (sg >> 1)) * kPageTokens + (sg & 1) * kStageKeys + warp * kWarpKeys;
        const int wkey = warp * kWarpKeys;  // first key of this warp within the stage

        // The score tile's column n of n-tile t is key wkey + 8t + kperm(n): the
        // eight keys of a column half-range sit at even / odd rows, so the K
        // operand loads of a half warp hit distinct banks of the swizzled rows.
        // This lane's keys (columns 2q + j) are wkey + 8t + k0 / k1.
        const int k0 = 2 * ((2 * q) & 3) + ((2 * q) >> 2), k1 = 2 * ((2 * q + 1) & 3) + ((2 * q + 1) >> 2);
        // K / V scale of block blk of this lane's keys of n-tile t, as a pair (j = 0, 1)
        auto scales = [&](int off, int t, int blk) {
            const __half* h0 = reinterpret_cast<const __half*>(sb + off + (wkey + 8 * t + k0) * (kBlocks * 2));
            const __half* h1 = reinterpret_cast<const __half*>(sb + off + (wkey + 8 * t + k1) * (kBlocks * 2));
            return make_float2(__half2float(h0[blk]), __half2float(h1[blk]));
        };

        // ---- QK^T ----
        float sc[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
        const uint8_t* kst = sb + kStageKq;
        if constexpr (KT == kKF16) {
            // f16 K: the stage holds each key as two 128-byte rows (dims 0..63,
            // 64..127), row 2 key + dims/64, swizzled like the int8 rows; the
            // lane's operand is the 8 values of dims 32 blk + 8q .. + 7, exact
#pragma unroll 1
            for (int blk = 0; blk < kBlocks; ++blk) {
                const uint4 qb = qfrag[32 * blk];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int key = wkey + 8 * t + 2 * (g & 3) + (g >> 2);
                    const int row = 2 * key + (blk >> 1), chunk = 4 * (blk & 1) + q;
                    const uint4 w = *reinterpret_cast<const uint4*>(kst + row * 128 + ((chunk ^ (row & 7)) << 4));
                    float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    mma16816(c, qb.x, qb.y, w.x, w.y);
                    mma16816(c, qb.z, qb.w, w.z, w.w);
                    sc[t][0] += c[0];
                    sc[t][1] += c[1];
                }
            }
        } else
#pragma unroll 1
        for (int blk = 0; blk < kBlocks; ++blk) {
            const uint4 qb = qfrag[32 * blk];  // k-steps 2 blk (x, y) and 2 blk + 1 (z, w)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int key = wkey + 8 * t + 2 * (g & 3) + (g >> 2);  // this lane's column of the K operand
                const int chunk = 2 * blk + (q >> 1);
                const uint2 w = *reinterpret_cast<const uint2*>(kst + key * kHeadDim + ((chunk ^ (key & 7)) << 4) +
                                                                8 * (q & 1));
                const uint32_t x0 = w.x ^ 0x80808080u, x1 = w.y ^ 0x80808080u;
                float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma16816(c, qb.x, qb.y,
                         h2u(__hsub2(u2h(__byte_perm(x0, 0x6464u, 0x5140u)), b1152)),
                         h2u(__hsub2(u2h(__byte_perm(x0, 0x6464u, 0x5342u)), b1152)));
                mma16816(c, qb.z, qb.w,
                         h2u(__hsub2(u2h(__byte_perm(x1, 0x6464u, 0x5140u)), b1152)),
                         h2u(__hsub2(u2h(__byte_perm(x1, 0x6464u, 0x5342u)), b1152)));
                const float2 kd = scales(kStageKd, t, blk);
                sc[t][0] = fmaf(kd.x, c[0], sc[t][0]);
                sc[t][1] = fmaf(kd.y, c[1], sc[t][1]);
            }
        }

        // ---- warp-local online softmax (log2 domain) for row g over the warp's 16 keys ----
        float sv[2][2];
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float v = (kbase + 8 * t + (j ? k1 : k0) <= kend) ? sc[t][j] * a.q_scale : -CUDART_INF_F;
                sv[t][j] = v;
                mx = fmaxf(mx, v);
            }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // the reference max moves only when the row's max exceeds it by more than 2^8
        const bool need = mx > m_run + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
            const float mn = need ? fmaxf(m_run, mx) : m_run;
            const float alpha = (mn == m_run) ? 1.0f : ex2_approx(m_run - mn);  // 0 when m_run was -inf
            m_run = mn;
            l_run *= alpha;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] *= alpha;
                o[nt][1] *= alpha;
            }
        }
        const float mu = (m_run == -CUDART_INF_F) ? 0.0f : m_run;
        float p[2][2];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                p[t][j] = ex2_approx(sv[t][j] - mu);  // 2^-inf = 0
                l_run += p[t][j];                       // this lane's share of the row sum
            }

        // ---- PV ----
        const uint8_t* vst = sb + kStageVq;
        // Q4_1 / Q5_1: A = p and B = the dequantized value fp16(q d + m), each
        // rounded once relative to itself (a separate fp32 sum of p m would
        // cancel against q d when the block minimum is large)
        uint32_t pp0 = 0u, pp1 = 0u;
        if constexpr (v_a_is_p(VT)) {
            pp0 = h2u(__floats2half2_rn(p[0][0], p[0][1]));
            pp1 = h2u(__floats2half2_rn(p[1][0], p[1][1]));
        }
        // the two keys' fp16 values of a per-(key, block) field, as a pair
        auto pair = [&](int off, int t, int blk) {
            const __half* h0 = reinterpret_cast<const __half*>(sb + off + (wkey + 8 * t + k0) * (kBlocks * 2));
            const __half* h1 = reinterpret_cast<const __half*>(sb + off + (wkey + 8 * t + k1) * (kBlocks * 2));
            return __halves2half2(h0[blk], h1[blk]);
        };
#pragma unroll
        for (int blk = 0; blk < kBlocks; ++blk) {
            // probabilities x the V scale of block blk, as the A operand
            uint32_t pa0, pa1;
            if constexpr (v_a_is_p(VT)) {
                pa0 = pp0;
                pa1 = pp1;
            } else {
                const float2 dv0 = scales(kStageVd, 0, blk), dv1 = scales(kStageVd, 1, blk);
                pa0 = h2u(__floats2half2_rn(p[0][0] * dv0.x, p[0][1] * dv0.y));
                pa1 = h2u(__floats2half2_rn(p[1][0] * dv1.x, p[1][1] * dv1.y));
            }
            // V code words of this lane's keys (k0, k1 of n-tiles 0 and 1): the
            // four codes of dims 32 blk + 4g + {0..3}
            uint32_t wv[2][2];
            // Q5_0: fifth bits of dims 32 blk + 4g + {0..3} of both keys of
            // n-tile t, in bits 0..3 (first key) and 16..19 (second key)
            uint32_t hv[2] = {0u, 0u};
            // F16: the four fp16 values of dims 32 blk + 4g + {0..3} of each key
            uint2 wf[2][2];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int key = wkey + 8 * t + (j ? k1 : k0);
                    if constexpr (VT == kVF16)
                        wf[t][j] = *reinterpret_cast<const uint2*>(vst + key * (kHeadDim * 2) + (32 * blk + 4 * g) * 2);
                    else if constexpr (VT == kVQ8_0)
                        wv[t][j] = *reinterpret_cast<const uint32_t*>(vst + key * kHeadDim + 32 * blk + 4 * g) ^
                                   0x80808080u;
                    else
                        wv[t][j] = *reinterpret_cast<const uint32_t*>(vst + key * 64 + 16 * blk + 4 * (g & 3));
                    if constexpr (v_has_fifth(VT))
                        hv[t] |= ((*reinterpret_cast<const uint32_t*>(sb + kStageVh + key * 16 + 4 * blk) >> (4 * g)) &
                                  0xfu) << (16 * j);
                }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t sel = (uint32_t)m | ((uint32_t)(4 + m) << 8);  // byte m of both words -> bytes 0, 2
                uint32_t bv[2];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if constexpr (VT == kVF16) {  // the two keys' values of dim 32 blk + 4g + m
                        const uint32_t a0 = (m < 2) ? wf[t][0].x : wf[t][0].y;
                        const uint32_t a1 = (m < 2) ? wf[t][1].x : wf[t][1].y;
                        bv[t] = __byte_perm(a0, a1, (m & 1) ? 0x7632u : 0x5410u);
                        continue;
                    }
                    const uint32_t pr = __byte_perm(wv[t][0], wv[t][1], sel);
                    if constexpr (VT == kVQ8_0)
                        bv[t] = h2u(__hsub2(u2h((pr & 0x00ff00ffu) | 0x64006400u), b1152));
                    else if constexpr (VT == kVQ5_0)  // 1024 + (nibble | fifth bit << 4) - 1040
                        bv[t] = h2u(__hsub2(u2h(((pr >> (4 * (g >> 2))) & 0x000f000fu) |
                                                (((hv[t] >> m) & 0x00010001u) << 4) | 0x64006400u),
                                            b1040));
                    else if constexpr (v_has_min(VT))  // fp16(q d + m), q = nibble (| fifth bit << 4)
                        bv[t] = h2u(__hfma2(__hsub2(u2h(((pr >> (4 * (g >> 2))) & 0x000f000fu) |
                                                        (((hv[t] >> m) & 0x00010001u) << 4) | 0x64006400u),
                                                    b1024),
                                            pair(kStageVd, t, blk), pair(kStageVm, t, blk)));
                    else
                        bv[t] = h2u(__hsub2(u2h(((pr >> (4 * (g >> 2))) & 0x000f000fu) | 0x64006400u), b1032));
                }
                float c[4] = {o[4 * blk + m][0], o[4 * blk + m][1], zr0, zr1};
                mma16816(c, pa0, pa1, bv[0], bv[1]);
                o[4 * blk + m][0] = c[0];
                o[4 * blk + m][1] = c[1];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[i % kStages]);  // this warp is done with the stage
    }
    ok = __syncthreads_and(ok);
    if (!ok) return;  // a bounded wait gave up; the error word is set

    // ---- merge the eight warps' (m, l, O) into the split's partial ----
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    float* red = reinterpret_cast<float*>(stage);          // [warps][ROWS][128]
    float* sml = red + kWarps * ROWS * kHeadDim;           // [warps][ROWS][2]
    if (g < ROWS) {
        float* dst = red + (warp * ROWS + g) * kHeadDim;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int d = 32 * (nt >> 2) + 8 * q + (nt & 3);  // columns 2q, 2q+1 -> dims d, d + 4
            dst[d] = o[nt][0];
            dst[d + 4] = o[nt][1];
        }
        if (q == 0) {
            sml[(warp * ROWS + g) * 2] = m_run;
            sml[(warp * ROWS + g) * 2 + 1] = l_run;
        }
    }
    __syncthreads();
    const int split_g = a.split_base + blockIdx.x;
    for (int idx = tid; idx < rows_here * kHeadDim; idx += kThreads) {
        const int r = idx / kHeadDim, d = idx - r * kHeadDim;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, sml[(ww * ROWS + r) * 2]);
        const float mu = (M == -CUDART_INF_F) ? 0.0f : M;
        float v = 0.0f, L = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
            const float wgt = ex2_approx(sml[(ww * ROWS + r) * 2] - mu);
            v = fmaf(wgt, red[(ww * ROWS + r) * kHeadDim + d], v);
            L = fmaf(wgt, sml[(ww * ROWS + r) * 2 + 1], L);
        }
        const int lr = row_begin + r;
        const int j = lr / a.group, g = lr - j * a.group;
        const int grow = j * a.n_qh + h * a.group + g;
        a.part.acc[((size_t)split_g * a.n_rows + grow) * kHeadDim + d] = v;
        if (d == 0) a.part.ml[(size_t)split_g * a.n_rows + grow] = make_float2(M, L);
    }
}

template <int ROWS, bool ZC, int VT, int KT>
static cudaError_t launch_decode_t(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                                   int n_row_groups, cudaStream_t s) {
    // the shared-memory opt-in is per device: remember which devices have it
    // devices whose shared-memory opt-in is done (calls from several host
    // threads may race to set a bit; the attribute call is idempotent)
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !(configured.load(std::memory_order_acquire) & (1ull << dev))) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<ROWS, ZC, VT, KT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)DecGeom<VT, KT>::kSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
    }
    dim3 grid(n_splits, a.n_kv, n_row_groups);
    decode_kernel<ROWS, ZC, VT, KT><<<grid, kThreads, DecGeom<VT, KT>::kSmem, s>>>(a, *kmap);
    return cudaGetLastError();
}

template <bool ZC, int VT, int KT = kKQ8_0>
static cudaError_t launch_decode_rows(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                                      cudaStream_t s) {
    const int rows = a.n_q * a.group;
    switch (rows) {
        case 1: return launch_decode_t<1, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        case 2: return launch_decode_t<2, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        case 3: return launch_decode_t<3, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        case 4: return launch_decode_t<4, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        case 5: return launch_decode_t<5, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        case 6: return launch_decode_t<6, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        case 7: return launch_decode_t<7, ZC, VT, KT>(a, kmap, n_splits, 1, s);
        default: return launch_decode_t<8, ZC, VT, KT>(a, kmap, n_splits, (rows + 7) / 8, s);
    }
}

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                          cudaStream_t s) {
    if (a.k_type == kKF16) return launch_decode_rows<false, kVF16, kKF16>(a, kmap, n_splits, s);
    if (a.v_type == kVQ8_0) return launch_decode_rows<false, kVQ8_0>(a, kmap, n_splits, s);
    if (a.v_type == kVQ5_0) return launch_decode_rows<false, kVQ5_0>(a, kmap, n_splits, s);
    if (a.v_type == kVQ4_1) return launch_decode_rows<false, kVQ4_1>(a, kmap, n_splits, s);
    if (a.v_type == kVQ5_1) return launch_decode_rows<false, kVQ5_1>(a, kmap, n_splits, s);
    if (a.v_type == kVF16) return launch_decode_rows<false, kVF16>(a, kmap, n_splits, s);
    return launch_decode_rows<false, kVQ4_0>(a, kmap, n_splits, s);
}

cudaError_t launch_decode_zero_copy(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                                    cudaStream_t s) {
    if (a.k_type == kKF16) return launch_decode_rows<true, kVF16, kKF16>(a, kmap, n_splits, s);
    if (a.v_type == kVQ8_0) return launch_decode_rows<true, kVQ8_0>(a, kmap, n_splits, s);
    if (a.v_type == kVQ5_0) return launch_decode_rows<true, kVQ5_0>(a, kmap, n_splits, s);
    if (a.v_type == kVQ4_1) return launch_decode_rows<true, kVQ4_1>(a, kmap, n_splits, s);
    if (a.v_type == kVQ5_1) return launch_decode_rows<true, kVQ5_1>(a, kmap, n_splits, s);
    if (a.v_type == kVF16) return launch_decode_rows<true, kVF16>(a, kmap, n_splits, s);
    return launch_decode_rows<true, kVQ4_0>(a, kmap, n_splits, s);
}

// ----------------------------------------------------------------------------
// K3: log-sum-exp merge.  CTA = (query row, 32-dim slice): M = max_s m_s,
// L = sum_s 2^(m_s-M) l_s, O = sum_s 2^(m_s-M) acc_s / L, lse = ln2 (M + log2 L).
// Warps stride over the splits with four independent loads in flight each.
// ----------------------------------------------------------------------------
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeArgs a) {
    __shared__ float sm[kMergeThreads / 32];
    __shared__ float sacc[kMergeThreads / 32][32];
    __shared__ float sl[kMergeThreads / 32];
    const int row = blockIdx.x;
    const int slice = blockIdx.y;  // dims [32 slice, 32 slice + 32)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int W = kMergeThreads / 32;
    if (a.err && *reinterpret_cast<const volatile int*>(a.err)) {  // a split's partial is missing
        if (warp == 0) {
            a.out[(size_t)row * kHeadDim + slice * 32 + lane] = CUDART_NAN_F;
            if (slice == 0 && lane == 0 && a.lse) a.lse[row] = CUDART_NAN_F;
        }
        return;
    }
    const float2* ml = a.part.ml + row;
    float m = -CUDART_INF_F;
    for (int s = tid; s < a.n_splits; s += kMergeThreads) m = fmaxf(m, ml[(size_t)s * a.n_rows].x);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) sm[warp] = m;
    __syncthreads();
    float M = sm[0];
#pragma unroll
    for (int w = 1; w < W; ++w) M = fmaxf(M, sm[w]);
    float L = 0.0f, o = 0.0f;
    const float* accp = a.part.acc + (size_t)row * kHeadDim + slice * 32 + lane;
    const size_t sstride = (size_t)a.n_rows * kHeadDim;
    int s = warp;
    for (; s + 3 * W < a.n_splits; s += 4 * W) {
        float2 mls[4];
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            mls[u] = ml[(size_t)(s + u * W) * a.n_rows];
            v[u] = accp[(size_t)(s + u * W) * sstride];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (mls[u].y > 0.0f) {
                const float w = exp2f(mls[u].x - M);
                L = fmaf(w, mls[u].y, L);
                o = fmaf(w, v[u], o);
            }
        }
    }
    for (; s < a.n_splits; s += W) {
        const float2 mlv = ml[(size_t)s * a.n_rows];
        const float v = accp[(size_t)s * sstride];
        if (mlv.y > 0.0f) {
            const float w = exp2f(mlv.x - M);
            L = fmaf(w, mlv.y, L);
            o = fmaf(w, v, o);
        }
    }
    sacc[warp][lane] = o;
    if (lane == 0) sl[warp] = L;
    __syncthreads();
    if (warp == 0) {
        float Lt = 0.0f, ot = 0.0f;
#pragma unroll
        for (int w = 0; w < W; ++w) { Lt += sl[w]; ot += sacc[w][lane]; }
        a.out[(size_t)row * kHeadDim + slice * 32 + lane] = ot / Lt;
        if (slice == 0 && lane == 0 && a.lse) a.lse[row] = (M + log2f(Lt)) * 0.69314718055994530942f;
    }
}

// Many query rows (verify / prefill chunks): one warp per row, lane = 4 dims,
// four splits in flight per lane; M first, then the weighted sums.
__global__ void __launch_bounds__(256) merge_rows_kernel(const MergeArgs a) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.n_rows) return;
    if (a.err && *reinterpret_cast<const volatile int*>(a.err)) {  // a split's partial is missing
        *reinterpret_cast<float4*>(a.out + (size_t)row * kHeadDim + 4 * lane) =
            make_float4(CUDART_NAN_F, CUDART_NAN_F, CUDART_NAN_F, CUDART_NAN_F);
        if (lane == 0 && a.lse) a.lse[row] = CUDART_NAN_F;
        return;
    }
    const float2* ml = a.part.ml + row;
    float m = -CUDART_INF_F;
    for (int s = lane; s < a.n_splits; s += 32) m = fmaxf(m, ml[(size_t)s * a.n_rows].x);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float* accp = a.part.acc + (size_t)row * kHeadDim + 4 * lane;
    const size_t sstride = (size_t)a.n_rows * kHeadDim;
    float L = 0.0f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    int s = 0;
    for (; s + 3 < a.n_splits; s += 4) {
        float2 mls[4];
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            mls[u] = ml[(size_t)(s + u) * a.n_rows];
            v[u] = *reinterpret_cast<const float4*>(accp + (size_t)(s + u) * sstride);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (mls[u].y > 0.0f) {
                const float w = exp2f(mls[u].x - m);
                L = fmaf(w, mls[u].y, L);
                o.x = fmaf(w, v[u].x, o.x); o.y = fmaf(w, v[u].y, o.y);
                o.z = fmaf(w, v[u].z, o.z); o.w = fmaf(w, v[u].w, o.w);
            }
        }
    }
    for (; s < a.n_splits; ++s) {
        const float2 mlv = ml[(size_t)s * a.n_rows];
        if (mlv.y > 0.0f) {
            const float4 v = *reinterpret_cast<const float4*>(accp + (size_t)s * sstride);
            const float w = exp2f(mlv.x - m);
            L = fmaf(w, mlv.y, L);
            o.x = fmaf(w, v.x, o.x); o.y = fmaf(w, v.y, o.y);
            o.z = fmaf(w, v.z, o.z); o.w = fmaf(w, v.w, o.w);
        }
    }
    const float inv = 1.0f / L;
    *reinterpret_cast<float4*>(a.out + (size_t)row * kHeadDim + 4 * lane) =
        make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    if (lane == 0 && a.lse) a.lse[row] = (m + log2f(L)) * 0.69314718055994530942f;
}

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s) {
    if (a.n_rows >= kMergeRowsMin) {
        merge_rows_kernel<<<(a.n_rows + 7) / 8, 256, 0, s>>>(a);
    } else {
        merge_kernel<<<dim3(a.n_rows, kHeadDim / 32), kMergeThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Self-test of the bounded wait: one thread waits on an mbarrier phase that
// nothing ever completes (no arrival, no transaction), through the same wait
// routine the kernels use, and must give up after limit_ns.
// ----------------------------------------------------------------------------
// small copies between pinned host memory and the device without the copy
// engines (whose queues the ring's chunk copies keep busy)
__global__ void __launch_bounds__(256) copy16_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                     size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

cudaError_t launch_copy16(void* dst, const void* src, size_t bytes, cudaStream_t s) {
    const size_t n = bytes / 16;
    if (n == 0) return cudaSuccess;
    const int blocks = (int)std::min<size_t>(64, (n + 255) / 256);
    copy16_kernel<<<blocks, 256, 0, s>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src), n);
    return cudaGetLastError();
}

__global__ void wait_selftest_kernel(int* err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait_bounded(&bar, 0, err, limit_ns);  // phase 0 never completes
}

cudaError_t launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t s) {
    wait_selftest_kernel<<<1, 1, 0, s>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace kvs

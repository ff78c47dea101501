// kvs_chunk_mma.cu -- K4: multi-token attention over quantized pages on the
// 5th-generation tensor cores (tcgen05), for speculative-verify batches and
// prefill chunks ("llama.cpp adaptive KV streaming - spec fork notes", Phase
// arena: speculative verify batches of 1 + n_draft tokens; 256-token ubatches
// on "RaymondHuang210129/llama.cpp-adaptive-kv-streaming", Summary).
//
// CTA = (split, kv head, 128-row M tile of the head's n_q x G query rows),
// 256 threads.  Per 128-key half-page stage of the split:
//   1. the raw Q8_0/Q4_0 stage lands in shared memory by TMA (same stage format
//      as the decode kernel; two stages in flight);
//   2. all threads dequantize it to fp16 UMMA operand tiles with the 128-byte
//      swizzle: K^ = d*q8 as [keys][dims] (K-major) split into two fp16 terms,
//      hi = fp16(d*q8) and lo = fp16(d*q8 - hi), whose sum is d*q8 to ~2^-22,
//      so the scores carry no fp16 rounding of K; V^ = fp16(d*(q4-8)) as
//      [keys][dims] (read by the MMA as an MN-major B operand);
//   3. one thread issues S = Q K^_hi^T + Q K^_lo^T (16 x tcgen05.mma M=128 N=128
//      K=16, f16 in, fp32 accumulate in tensor memory);
//   4. all eight warps (thread = query row = TMEM lane, two warps per row
//      splitting the 128 key columns) read S back, apply the causal mask, the
//      1/sqrt(128) scale in the log2 domain and the online softmax; P is
//      written as fp16 in the UMMA A layout.  A row keeps its reference max
//      until the row max exceeds it by more than 2^8 (p <= 256 stays exact
//      enough in fp16 and fp32 sums); only then is its O row in tensor memory
//      rescaled;
//   5. one thread issues O += P V^ (8 x tcgen05.mma).
// At the end O, m, l of every valid row are written as the split's partials,
// merged later by the LSE merge kernel.  No cluster, no multicast.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "kvs_internal.h"
#include "kvs_ptx.cuh"

namespace kvs {
namespace {

constexpr int kTcThreads = 256;
constexpr int kMTile = 128;
constexpr int kKeys = 128;  // keys per stage
constexpr int kRawKq = 0;
constexpr int kRawKd = kKeys * kHeadDim;                 // 16384
constexpr int kRawVq = kRawKd + kKeys * kBlocks * 2;     // 17408
constexpr int kRawVd = kRawVq + kKeys * kHeadDim / 2;    // 25600
constexpr int kRawBytes = kRawVd + kKeys * kBlocks * 2;  // 26624
constexpr int kRawStages = 2;
constexpr int kTileBytes = kMTile * kHeadDim * 2;        // 32768: 128 x 128 fp16
constexpr size_t kOffQ = (size_t)kRawStages * kRawBytes;  // 53248
constexpr size_t kOffK = kOffQ + kTileBytes;     // K^ high part
constexpr size_t kOffKlo = kOffK + kTileBytes;   // K^ low part
constexpr size_t kOffV = kOffKlo + kTileBytes;
constexpr size_t kOffP = kOffV + kTileBytes;
constexpr size_t kOffRowMax = kOffP + kTileBytes;  // [2 column halves][128 rows] fp32
constexpr size_t kOffBar = kOffRowMax + 2 * kMTile * 4;  // raw[2], s, o
constexpr size_t kOffTmem = kOffBar + 4 * 8;
constexpr size_t kTcSmem = 1024 + kOffTmem + 16;
constexpr uint32_t kTmemCols = 256;              // S: columns 0..127, O: 128..255
static_assert(kOffQ % 1024 == 0 && kRawBytes % 1024 == 0, "swizzled tiles need 1024-B alignment");

// instruction descriptor: f16 x f16 -> f32, M = 128, N = 128, A K-major,
// B K-major (QK^T) or MN-major (PV)
constexpr uint32_t kIdescQK = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 16);

// byte offset of element (row, col) of a 128 x 128 fp16 tile stored as two
// 64-column halves of 16 KB, rows of 128 B in 8-row groups of 1 KB, 16-byte
// chunks XOR-swizzled by the row within its group (the 128-byte swizzle)
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
    return (uint32_t)((col >> 6) * 16384 + (row >> 3) * 1024 + (row & 7) * 128 +
                      ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}

// shared-memory matrix descriptor (version 1, 128-byte swizzle)
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((start >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand (rows x 128 k), k-step kk of 16 elements
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int kk) {
    return smem_desc(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
}
// MN-major operand V^ [keys][dims]: 8-key groups 1 KB apart (K direction),
// 64-dim halves 16 KB apart (N direction); k-step kk covers keys 16kk..16kk+15
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int kk) {
    return smem_desc(base + kk * 2048, 16384, 1024);
}

// 2^x with the hardware approximation (flush-to-zero; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, so that half of the softmax exponentials leave the
// XU pipe (which the MUFU exponentials and fp16 packing saturate): x = n + f
// with n the nearest integer (1.5 * 2^23 rounding trick) and f in [-0.5, 0.5];
// 2^f from a degree-5 polynomial fitted by weighted least squares (Lawson
// iterations) to 2^f on [-0.5, 0.5], max relative error 2.4e-7 in binary32;
// 2^n added to the exponent field.  x <= -127 gives +0.
__device__ __forceinline__ float exp2_poly(float x) {
    x = fmaxf(x, -127.0f);
    const float rn = x + 12582912.0f;
    const float n = rn - 12582912.0f;
    const float f = x - n;
    float p = 0.001327646430581808f;
    p = fmaf(p, f, 0.009675540961325169f);
    p = fmaf(p, f, 0.05550713464617729f);
    p = fmaf(p, f, 0.24022120237350464f);
    p = fmaf(p, f, 0.6931469440460205f);
    p = fmaf(p, f, 1.0000001192092896f);
    const int e = __float_as_int(rn) - 0x4B400000;
    return __int_as_float(__float_as_int(p) + (e << 23));
}

__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

__global__ void __launch_bounds__(kTcThreads, 1)
    chunk_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* raw = smem;
    uint8_t* sQ = smem + kOffQ;
    uint8_t* sK = smem + kOffK;
    uint8_t* sKlo = smem + kOffKlo;
    uint8_t* sV = smem + kOffV;
    uint8_t* sP = smem + kOffP;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.y;
    const int rows_head = a.n_q * a.group;
    const int st0 = (int)(((long)blockIdx.x * 2 * a.n_units) / a.n_splits);
    const int n_st = (int)(((long)(blockIdx.x + 1) * 2 * a.n_units) / a.n_splits) - st0;

    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (int b = 0; b < 4; ++b) mbar_init(&bar[b], 1);
        fence_mbar_init();
    }
    // Q tile: row r = local query row mt*128 + r (rows past the head's rows are zero)
    for (int idx = tid; idx < kMTile * 16; idx += kTcThreads) {
        const int r = idx >> 4, c = idx & 15;
        const int lr = blockIdx.z * kMTile + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (lr < rows_head) {
            const int j = lr / a.group, g = lr - j * a.group;
            v = *reinterpret_cast<const uint4*>(a.q + ((size_t)j * a.n_qh + h * a.group + g) * kHeadDim + c * 8);
        }
        *reinterpret_cast<uint4*>(sQ + tile_off(r, c * 8)) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = *tmem_slot;
    const uint32_t t_s = taddr, t_o = taddr + 128;

    auto issue = [&](int i) {
        const int sg = st0 + i;
        const int u = sg >> 1, half = sg & 1;
        const int slot = (a.slot0 + u) % a.region_slots;
        const uint8_t* ph = a.region + ((size_t)slot * a.n_kv + h) * kPageHeadBytes;
        uint8_t* dst = raw + (i & 1) * kRawBytes;
        uint64_t* b = &bar[i & 1];
        mbar_expect_tx(b, kRawBytes);
        const int krow = ((a.region_slot_base + slot) * a.n_kv + h) * kPageHeadRows + half * kKeys;
        tma_load_2d(dst + kRawKq, &kmap, 0, krow, b);
        bulk_load(dst + kRawKd, ph + kOffKd + half * (kKeys * kBlocks * 2), kKeys * kBlocks * 2, b);
        bulk_load(dst + kRawVq, ph + kOffVq + half * (kKeys * kHeadDim / 2), kKeys * kHeadDim / 2, b);
        bulk_load(dst + kRawVd, ph + kOffVd + half * (kKeys * kBlocks * 2), kKeys * kBlocks * 2, b);
    };
    if (tid == 0) {
        for (int i = 0; i < kRawStages && i < n_st; ++i) issue(i);
    }

    // softmax role: every warp takes one 32-row quarter of the tile (its TMEM
    // lane quarter) and one half of the 128 key columns: warp w -> rows
    // 32 (w % 4) .. +32, columns 64 (w / 4) .. +64.
    const int srow = (warp & 3) * 32 + (tid & 31);
    const int chalf = warp >> 2;
    const int lrow = blockIdx.z * kMTile + srow;
    const bool row_valid = lrow < rows_head;
    const bool warp_active = __any_sync(0xffffffffu, row_valid);
    const int qpos = row_valid ? a.pos0 + lrow / a.group : -1;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float m_ref = -CUDART_INF_F, l_part = 0.0f;  // l_part: this thread's column half
    float* sRowMax = reinterpret_cast<float*>(smem + kOffRowMax);  // [2][128]
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aKlo = smem_u32(sKlo), aV = smem_u32(sV),
                   aP = smem_u32(sP);
    bool ok = true;
    for (int i = 0; i < n_st; ++i) {
        const int sg = st0 + i;
        const uint8_t* rb = raw + (i & 1) * kRawBytes;
        if (!mbar_wait_bounded(&bar[i & 1], (i >> 1) & 1, a.err)) ok = false;
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---- dequantize K^ (K-major [keys][dims]) ----
        {
            const int key = tid & 127;
            for (int g = tid >> 7; g < 8; g += 2) {  // 16-dim chunk g of the key's row
                const uint4 q = *reinterpret_cast<const uint4*>(rb + kRawKq + key * 128 + ((g ^ (key & 7)) << 4));
                const __half dh = *reinterpret_cast<const __half*>(rb + kRawKd + key * 8 + (g >> 1) * 2);
                const __half2 d2 = __halves2half2(dh, dh);
                const __half2 bias = __float2half2_rn(1152.0f);
                const uint32_t w[4] = {q.x ^ 0x80808080u, q.y ^ 0x80808080u, q.z ^ 0x80808080u,
                                       q.w ^ 0x80808080u};
                uint32_t o[8], ol[8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    // bytes (0,1) and (2,3) -> fp16 1024 + 128 + x, exact; minus 1152 -> x;
                    // hi = fp16(x d); lo = fp16(x d - hi) (the FMA forms x d - hi exactly)
                    const __half2 x01 = __hsub2(u2h(__byte_perm(w[u], 0x6464u, 0x5140u)), bias);
                    const __half2 x23 = __hsub2(u2h(__byte_perm(w[u], 0x6464u, 0x5342u)), bias);
                    const __half2 h01 = __hmul2(x01, d2), h23 = __hmul2(x23, d2);
                    o[2 * u] = h2u(h01);
                    o[2 * u + 1] = h2u(h23);
                    ol[2 * u] = h2u(__hfma2(x01, d2, __hneg2(h01)));
                    ol[2 * u + 1] = h2u(__hfma2(x23, d2, __hneg2(h23)));
                }
                *reinterpret_cast<uint4*>(sK + tile_off(key, g * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(sK + tile_off(key, g * 16 + 8)) = make_uint4(o[4], o[5], o[6], o[7]);
                *reinterpret_cast<uint4*>(sKlo + tile_off(key, g * 16)) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                *reinterpret_cast<uint4*>(sKlo + tile_off(key, g * 16 + 8)) = make_uint4(ol[4], ol[5], ol[6], ol[7]);
            }
        }
        // ---- dequantize V^ ([keys][dims]; block b of a key: byte j = dims 32b+j (low), 32b+16+j (high)) ----
        for (int un = tid; un < kKeys * kBlocks; un += kTcThreads) {
            const int b = un & 3, key = un >> 2;
            const uint4 q = *reinterpret_cast<const uint4*>(rb + kRawVq + key * 64 + b * 16);
            const __half dh = *reinterpret_cast<const __half*>(rb + kRawVd + key * 8 + b * 2);
            const __half2 d2 = __halves2half2(dh, dh);
            const __half2 bias = __float2half2_rn(1032.0f);
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
            uint32_t lo[8], hi[8];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t p01 = __byte_perm(w[u], 0u, 0x4140u);  // bytes 4u, 4u+1 at positions 0, 2
                const uint32_t p23 = __byte_perm(w[u], 0u, 0x4342u);
                lo[2 * u] = h2u(__hmul2(__hsub2(u2h((p01 & 0x000F000Fu) | 0x64006400u), bias), d2));
                lo[2 * u + 1] = h2u(__hmul2(__hsub2(u2h((p23 & 0x000F000Fu) | 0x64006400u), bias), d2));
                hi[2 * u] = h2u(__hmul2(__hsub2(u2h(((p01 >> 4) & 0x000F000Fu) | 0x64006400u), bias), d2));
                hi[2 * u + 1] = h2u(__hmul2(__hsub2(u2h(((p23 >> 4) & 0x000F000Fu) | 0x64006400u), bias), d2));
            }
            *reinterpret_cast<uint4*>(sV + tile_off(key, 32 * b)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            *reinterpret_cast<uint4*>(sV + tile_off(key, 32 * b + 8)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            *reinterpret_cast<uint4*>(sV + tile_off(key, 32 * b + 16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sV + tile_off(key, 32 * b + 24)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        }
        fence_proxy_async_smem();
        __syncthreads();
        // the raw buffer is consumed: refill it with stage i + 2
        if (tid == 0 && i + kRawStages < n_st) issue(i + kRawStages);

        // ---- S = Q K^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) tc_mma_f16(t_s, desc_k(aQ, kk), desc_k(aK, kk), kIdescQK, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) tc_mma_f16(t_s, desc_k(aQ, kk), desc_k(aKlo, kk), kIdescQK, 1u);
            tc_commit(&bar[2]);
        }

        // ---- online softmax on the tensor-memory S rows ----
        if (!mbar_wait_bounded(&bar[2], i & 1, a.err)) ok = false;
        tc_fence_after();
        float v[64];
        const int kbase = (a.page0 + (sg >> 1)) * kPageTokens + (sg & 1) * kKeys + chalf * 64;
        const int kend = min(a.len - 1, qpos);  // last visible key position of this row
        if (warp_active) {
            float mx = -CUDART_INF_F;
            float tmp[32];
            tmem_ld32(t_s + lane_off + chalf * 64, tmp);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = tmp[e];
            tmem_ld32(t_s + lane_off + chalf * 64 + 32, tmp);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[32 + e] = tmp[e];
            if (kbase + 63 <= kend) {
#pragma unroll
                for (int e = 0; e < 64; ++e) mx = fmaxf(mx, v[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    if (kbase + e > kend) v[e] = -CUDART_INF_F;
                    mx = fmaxf(mx, v[e]);
                }
            }
            sRowMax[chalf * kMTile + srow] = mx;
        }
        __syncthreads();
        if (warp_active) {
            // scores in the log2 domain are v * q_scale (q_scale > 0)
            const float m_stage = fmaxf(sRowMax[srow], sRowMax[kMTile + srow]) * a.q_scale;
            // keep the reference max unless the row's max grew by more than 2^8
            float m_use = m_ref;
            if (m_stage > m_ref + 8.0f) m_use = m_stage;
            const float mu = (m_use == -CUDART_INF_F) ? 0.0f : m_use;
            const float alpha = (m_use == m_ref) ? 1.0f : ex2_approx(m_ref - mu);
            m_ref = m_use;
            l_part *= alpha;
            if (i > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                float o[32];
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    tmem_ld32(t_o + lane_off + chalf * 64 + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tmem_st32(t_o + lane_off + chalf * 64 + c * 32, o);
                }
            }
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                const float p0 = ex2_approx(fmaf(v[e], a.q_scale, -mu));      // 2^-inf = 0
                const float p1 = exp2_poly(fmaf(v[e + 1], a.q_scale, -mu));
                l_part += p0 + p1;
                pk[e >> 1] = h2u(__floats2half2_rn(p0, p1));
            }
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
                *reinterpret_cast<uint4*>(sP + tile_off(srow, chalf * 64 + q4 * 8)) =
                    make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---- O += P V^ ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc_mma_f16(t_o, desc_k(aP, kk), desc_mn(aV, kk), kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&bar[3]);
        }
        if (!mbar_wait_bounded(&bar[3], i & 1, a.err)) ok = false;
        tc_fence_after();
    }

    // ---- write the split's partials: each warp its rows' column half of O ----
    ok = __syncthreads_and(ok);
    if (ok) {
        float* sL = reinterpret_cast<float*>(smem + kOffRowMax);  // reuse: [2][128]
        sL[chalf * kMTile + srow] = l_part;
        __syncthreads();
        const int split_g = a.split_base + blockIdx.x;
        const int j = lrow / a.group, g = lrow - j * a.group;
        const int grow = j * a.n_qh + h * a.group + g;
        if (warp_active) {
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                float o[32];
                tmem_ld32(t_o + lane_off + chalf * 64 + c * 32, o);
                if (row_valid) {
                    float* dst = a.part.acc + ((size_t)split_g * a.n_rows + grow) * kHeadDim + chalf * 64 + c * 32;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
                }
            }
        }
        if (row_valid && chalf == 0)
            a.part.ml[(size_t)split_g * a.n_rows + grow] = make_float2(m_ref, sL[srow] + sL[kMTile + srow]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(taddr, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_chunk_mma(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits, cudaStream_t s) {
    static unsigned long long configured = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !(configured & (1ull << dev))) {
        cudaError_t e = cudaFuncSetAttribute(chunk_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kTcSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured |= 1ull << dev;
    }
    const int m_tiles = (a.n_q * a.group + kMTile - 1) / kMTile;
    dim3 grid(n_splits, a.n_kv, m_tiles);
    chunk_mma_kernel<<<grid, kTcThreads, kTcSmem, s>>>(a, *kmap);
    return cudaGetLastError();
}

}  // namespace kvs

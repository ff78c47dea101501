// kvs_static.cu -- kvs_attend_pages_static: attention over caller-owned,
// device-resident quantized pages that performs no device allocation.
//
// Why it exists: some callers cannot call cudaMalloc on their hot path.  An
// engine that owns every byte of device memory through its own pool, a caller
// whose allocations are frozen after start-up (so that nothing can fail for
// lack of memory mid-request), or a latency-critical loop that must not take
// cudaMalloc's implicit device synchronization all need the attention step to
// run without asking the CUDA runtime for memory.  The handle-based kvs_attend
// allocates its scratch once in kvs_create; this entry point instead keeps its
// scratch (the per-split softmax partials) in one fixed-size static __device__
// array of this library, so no handle and no allocation are needed at all.
//
// The array is shared by every call on a device and keeps the previous call's
// contents.  The partials need no clearing: the split kernel writes every
// (split, row) record that the merge kernel then reads.  One record can be
// missing only if a split kernel's bounded wait gives up; that sets a static
// error word, which each call clears first (a 4-byte cudaMemsetAsync, no
// allocation), and the merge then writes NaN instead of reading stale records.
// Two calls whose kernels overlap on the GPU (different streams without
// ordering between them) race on the array; callers must order such calls.
#include <mutex>

#include "../../include/kvs.h"
#include "kvs_internal.h"

using namespace kvs;

namespace {

constexpr int kStaticMaxSplits = 64;
constexpr int kStaticMaxRows = 64;  // n_q * n_q_heads
constexpr size_t kStaticAccFloats = (size_t)kStaticMaxSplits * kStaticMaxRows * kHeadDim;
constexpr size_t kStaticFloats = kStaticAccFloats + (size_t)kStaticMaxSplits * kStaticMaxRows * 2;

// 2 MiB + 32 KiB per device, held by every GPU that loads the library until exit
static __device__ __align__(256) float g_static_scratch[kStaticFloats];
// set by a split kernel whose bounded wait gave up; cleared at the start of each call
static __device__ int g_static_err;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
float* g_scratch_addr[64] = {};  // device address of g_static_scratch, per device
int* g_err_addr[64] = {};        // device address of g_static_err, per device
EncodeTiledFn g_encode = nullptr;

int fail(int code, const char* msg) {
    set_last_error(msg);  // read back with kvs_last_error(NULL)
    return code;
}

// Once per device, with that device current: look up the array's device address
// (the host-side symbol is only a stand-in and must never reach a kernel).
int setup(int dev, float** scratch, int** err) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev < 0 || dev >= 64) return fail(KVS_E_INVAL, "device index out of range");
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        void* pe = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p) return fail(KVS_E_CUDA, "cudaGetSymbolAddress(scratch) failed");
        e = cudaGetSymbolAddress(&pe, g_static_err);
        if (e != cudaSuccess || !pe) return fail(KVS_E_CUDA, "cudaGetSymbolAddress(error word) failed");
        g_err_addr[dev] = static_cast<int*>(pe);
        g_scratch_addr[dev] = static_cast<float*>(p);
    }
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr);
        if (e != cudaSuccess || qr != cudaDriverEntryPointSuccess || !fn)
            return fail(KVS_E_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    *scratch = g_scratch_addr[dev];
    *err = g_err_addr[dev];
    return KVS_OK;
}

}  // namespace

extern "C" int kvs_attend_pages_static(const void* pages, int n_pages, int n_tokens, int n_q_heads,
                                       int n_kv_heads, int pos0, int n_q, const void* q_f16,
                                       float* out, float* lse, void* stream) {
    if (!pages || !q_f16 || !out) return fail(KVS_E_INVAL, "null pages/q/out");
    if (n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads != 0)
        return fail(KVS_E_INVAL, "n_q_heads must be a positive multiple of n_kv_heads");
    if (n_tokens < 1 || n_pages < (n_tokens + kPageTokens - 1) / kPageTokens)
        return fail(KVS_E_INVAL, "n_pages does not cover n_tokens");
    if (n_q < 1 || pos0 < 0 || (long)pos0 + n_q > n_tokens)
        return fail(KVS_E_ORDER, "queries must lie inside the n_tokens history");
    if ((long)n_q * n_q_heads > kStaticMaxRows)
        return fail(KVS_E_WIDTH, "n_q * n_q_heads exceeds the static scratch maximum of 64 rows");
    // the kernels' vector accesses: pages by TMA and 16-byte copies, Q in
    // 8-byte words, out and lse as single floats
    if (reinterpret_cast<uintptr_t>(pages) & 15) return fail(KVS_E_INVAL, "pages must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(q_f16) & 7) return fail(KVS_E_INVAL, "q must be 8-byte aligned");
    if ((reinterpret_cast<uintptr_t>(out) & 3) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return fail(KVS_E_INVAL, "out and lse must be 4-byte aligned");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVS_E_CUDA, "cudaGetDevice failed");
    float* scratch = nullptr;
    int* err = nullptr;
    int rc = setup(dev, &scratch, &err);
    if (rc != KVS_OK) return rc;

    const int used_pages = (n_tokens + kPageTokens - 1) / kPageTokens;
    const uint64_t rows_2d = (uint64_t)used_pages * n_kv_heads * kPageHeadRows;
    CUtensorMap kmap;
    cuuint64_t dims[2] = {128, rows_2d};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    if (g_encode(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(pages), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return fail(KVS_E_CUDA, "cuTensorMapEncodeTiled failed");

    const int rows = n_q * n_q_heads;
    const int stages = 2 * used_pages;
    const int sps = (stages + kStaticMaxSplits - 1) / kStaticMaxSplits;
    const int n_splits = (stages + sps - 1) / sps;

    DecodeArgs d{};
    d.v_type = kVQ4_0;  // caller pages use the K Q8_0 / V Q4_0 page layout
    d.region = static_cast<const uint8_t*>(pages);
    d.region_slot_base = 0;
    d.region_slots = used_pages;
    d.slot0 = 0;
    d.page0 = 0;
    d.n_units = used_pages;
    d.n_splits = n_splits;
    d.split_base = 0;
    d.len = n_tokens;
    d.pos0 = pos0;
    d.n_q = n_q;
    d.q = static_cast<const __half*>(q_f16);
    d.q_scale = (float)(1.4426950408889634 / 11.313708498984761);  // log2(e)/sqrt(128)
    d.n_qh = n_q_heads;
    d.n_kv = n_kv_heads;
    d.group = n_q_heads / n_kv_heads;
    d.part.acc = scratch;
    d.part.ml = reinterpret_cast<float2*>(scratch + kStaticAccFloats);
    d.n_rows = rows;
    d.err = err;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
    if (e != cudaSuccess) return fail(KVS_E_CUDA, cudaGetErrorString(e));
    e = launch_decode(d, &kmap, n_splits, s);
    if (e != cudaSuccess) return fail(KVS_E_CUDA, cudaGetErrorString(e));
    MergeArgs m;
    m.part = d.part;
    m.n_splits = n_splits;
    m.n_rows = rows;
    m.out = out;
    m.lse = lse;
    m.err = err;
    e = launch_merge(m, s);
    if (e != cudaSuccess) return fail(KVS_E_CUDA, cudaGetErrorString(e));
    return KVS_OK;
}

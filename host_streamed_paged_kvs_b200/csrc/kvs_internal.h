// kvs_internal.h -- layout constants and kernel launcher declarations shared by
// the host runtime (kvs_runtime.cpp) and the sm_100a kernels (kvs_kernels.cu,
// kvs_chunk_mma.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvs {

// ---------------------------------------------------------------------------
// Page layout in HBM and in pinned host memory (identical bytes on both sides).
//
// One page = 256 tokens of one layer, all kv heads: [n_kv][page_head].  One
// page_head (53,248 B) is split by field so that every field is 16-byte
// aligned and a 128-token half page of each field is contiguous:
//   Kq  int8  [256 tok][128 dims]                 32,768 B  @ 0
//   Kd  fp16  [256 tok][4 blocks]                   2,048 B  @ 32,768
//   Vq  u8    [256 tok][4 blocks][16 B]            16,384 B  @ 34,816
//         (byte j of a block holds code j in the low nibble, code j+16 high)
//   Vd  fp16  [256 tok][4 blocks]                   2,048 B  @ 51,200
// The canonical blocks (34-byte Q8_0, 18-byte Q4_0 and the V types below)
// are a reshuffle of these bytes (kvs_export_page does it on the host).
// ---------------------------------------------------------------------------
constexpr int kHeadDim = 128;
constexpr int kPageTokens = 256;
constexpr int kBlocks = kHeadDim / 32;                  // 4
constexpr int kOffKq = 0;
constexpr int kOffKd = kPageTokens * kHeadDim;          // 32768
constexpr int kOffVq = kOffKd + kPageTokens * kBlocks * 2;  // 34816
constexpr int kOffVd = kOffVq + kPageTokens * kHeadDim / 2;  // 51200
constexpr int kPageHeadBytes = kOffVd + kPageTokens * kBlocks * 2;  // 53248
constexpr int kPageHeadRows = kPageHeadBytes / 128;     // 416 rows of 128 B
static_assert(kPageHeadBytes == 53248, "page-head layout");

// K type codes (the public KVS_TYPE_* values): Q8_0, or F16 (the f16-f16 pair)
constexpr int kKF16 = 1;
constexpr int kKQ8_0 = 8;

// V type codes (the public KVS_TYPE_* values)
constexpr int kVF16 = 1;
constexpr int kVQ4_0 = 2;
constexpr int kVQ4_1 = 3;
constexpr int kVQ5_0 = 6;
constexpr int kVQ5_1 = 7;
constexpr int kVQ8_0 = 8;

// V type traits: fifth code bit (Q5_x), block minimum (Q4_1, Q5_1), levels
__host__ __device__ constexpr bool v_has_fifth(int vt) { return vt == kVQ5_0 || vt == kVQ5_1; }
__host__ __device__ constexpr bool v_has_min(int vt) { return vt == kVQ4_1 || vt == kVQ5_1; }
// decode feeds the tensor cores p and the V value itself (no per-block scale in A)
__host__ __device__ constexpr bool v_a_is_p(int vt) { return v_has_min(vt) || vt == kVF16; }

// Page-head geometry by V type.  Q4_0 V is the layout above.  Q8_0 V stores
// its codes like K (int8 [256 tok][128 dims], block b = dims 32b..32b+31):
//   Kq @ 0, Kd @ 32,768, Vq int8 [256][128] @ 34,816, Vd @ 67,584; 69,632 B.
// The other types keep the low 4 bits of their codes as Q4_0 keeps its codes;
// Q5_x add the fifth bits, one 32-bit word per block (bit j = code j's bit 4),
// and Q4_1 / Q5_1 the block minimum m (fp16) after the scales:
//   Q5_0: Vq @ 34,816, Vh u32 [256][4] @ 51,200, Vd @ 55,296; 57,344 B.
//   Q4_1: Vq @ 34,816, Vd @ 51,200, Vm fp16 [256][4] @ 53,248; 55,296 B.
//   Q5_1: Vq @ 34,816, Vh @ 51,200, Vd @ 55,296, Vm @ 57,344; 59,392 B.
// F16 V stores the values, fp16 [256 tok][128 dims] @ 34,816, and no scales;
// 100,352 B.
// F16 K (only with F16 V: the f16-f16 pair) stores the K values the same way,
// fp16 [256 tok][128 dims] @ 0, and no K scales; V then starts at 65,536 and
// the page head is 131,072 B.
template <int VT, int KT = kKQ8_0>
struct PageGeom {
    static_assert(VT == kVF16 || VT == kVQ4_0 || VT == kVQ4_1 || VT == kVQ5_0 || VT == kVQ5_1 || VT == kVQ8_0,
                  "V type");
    static_assert(KT == kKQ8_0 || (KT == kKF16 && VT == kVF16), "K/V type pair");
    static constexpr int kKqRow = KT == kKF16 ? kHeadDim * 2 : kHeadDim;  // K bytes per token
    static constexpr int kKdRow = KT == kKF16 ? 0 : kBlocks * 2;          // K scale bytes per token
    static constexpr int kOffKq = 0;
    static constexpr int kOffKd = kPageTokens * kKqRow;                    // 32768 for Q8_0 K
    static constexpr int kVqRow =                                           // V code bytes per token
        VT == kVQ8_0 ? kHeadDim : (VT == kVF16 ? kHeadDim * 2 : kHeadDim / 2);
    static constexpr int kVhRow = v_has_fifth(VT) ? kBlocks * 4 : 0;      // V fifth-bit bytes per token
    static constexpr int kVdRow = VT == kVF16 ? 0 : kBlocks * 2;          // V scale bytes per token
    static constexpr int kVmRow = v_has_min(VT) ? kBlocks * 2 : 0;        // V minimum bytes per token
    static constexpr int kOffVq = kOffKd + kPageTokens * kKdRow;           // 34816 for Q8_0 K
    static constexpr int kOffVh = kOffVq + kPageTokens * kVqRow;
    static constexpr int kOffVd = kOffVh + kPageTokens * kVhRow;
    static constexpr int kOffVm = kOffVd + kPageTokens * kVdRow;
    static constexpr int kHeadBytes = kOffVm + kPageTokens * kVmRow;
    static constexpr int kRows = kHeadBytes / 128;
    static constexpr int kLevels = VT == kVQ4_1 ? 15 : 31;                // Q4_1 / Q5_1 steps
    static constexpr int kVBlockBytes =                                    // canonical block
        VT == kVQ8_0 ? 34
                     : (VT == kVQ5_0 ? 22 : (VT == kVQ4_1 ? 20 : (VT == kVQ5_1 ? 24 : (VT == kVF16 ? 64 : 18))));
};
static_assert(PageGeom<kVQ4_0>::kHeadBytes == kPageHeadBytes && PageGeom<kVQ4_0>::kOffVd == kOffVd,
              "Q4_0 geometry");
static_assert(PageGeom<kVQ8_0>::kHeadBytes == 69632 && PageGeom<kVQ8_0>::kHeadBytes % 128 == 0,
              "Q8_0 geometry");
static_assert(PageGeom<kVQ5_0>::kHeadBytes == 57344 && PageGeom<kVQ5_0>::kOffVh == 51200 &&
                  PageGeom<kVQ5_0>::kOffVd == 55296 && PageGeom<kVQ5_0>::kHeadBytes % 128 == 0,
              "Q5_0 geometry");
static_assert(PageGeom<kVQ4_1>::kHeadBytes == 55296 && PageGeom<kVQ4_1>::kOffVd == 51200 &&
                  PageGeom<kVQ4_1>::kOffVm == 53248 && PageGeom<kVQ4_1>::kHeadBytes % 128 == 0,
              "Q4_1 geometry");
static_assert(PageGeom<kVF16>::kHeadBytes == 100352 && PageGeom<kVF16>::kHeadBytes % 128 == 0, "F16 geometry");
static_assert(PageGeom<kVF16, kKF16>::kHeadBytes == 131072 && PageGeom<kVF16, kKF16>::kOffVq == 65536,
              "F16-F16 geometry");
static_assert(PageGeom<kVQ5_1>::kHeadBytes == 59392 && PageGeom<kVQ5_1>::kOffVh == 51200 &&
                  PageGeom<kVQ5_1>::kOffVd == 55296 && PageGeom<kVQ5_1>::kOffVm == 57344 &&
                  PageGeom<kVQ5_1>::kHeadBytes % 128 == 0,
              "Q5_1 geometry");
inline int page_head_bytes(int v_type, int k_type = kKQ8_0) {
    if (k_type == kKF16) return PageGeom<kVF16, kKF16>::kHeadBytes;
    switch (v_type) {
        case kVQ8_0: return PageGeom<kVQ8_0>::kHeadBytes;
        case kVQ5_0: return PageGeom<kVQ5_0>::kHeadBytes;
        case kVQ4_1: return PageGeom<kVQ4_1>::kHeadBytes;
        case kVQ5_1: return PageGeom<kVQ5_1>::kHeadBytes;
        case kVF16: return PageGeom<kVF16>::kHeadBytes;
        default: return PageGeom<kVQ4_0>::kHeadBytes;
    }
}
inline bool v_type_supported(int v_type) {
    return v_type == kVF16 || v_type == kVQ4_0 || v_type == kVQ4_1 || v_type == kVQ5_0 || v_type == kVQ5_1 ||
           v_type == kVQ8_0;
}
// the K/V pairs the kernels are built for: K Q8_0 with every V type, and f16-f16
inline bool kv_pair_supported(int k_type, int v_type) {
    return (k_type == kKQ8_0 && v_type_supported(v_type)) || (k_type == kKF16 && v_type == kVF16);
}

// split partials: per split and query row, (m, l) in the log2 domain + acc[128]
struct PartialBuffers {
    float2* ml;   // [n_splits][n_rows]
    float* acc;   // [n_splits][n_rows][128]
};

struct AppendArgs {
    const __half* k;         // [n_tok][n_kv][128]
    const __half* v;
    uint8_t* host_layer;     // device alias of the layer's host history (page 0)
    uint8_t* res_layer;      // layer's resident region (slot 0)
    int n_tok, pos0, n_kv;
    int n_resident;          // R
    int first_resident_page; // pages >= this are resident after the append
    size_t page_bytes;
    int v_type;              // V type (kV*)
    int k_type;              // K type (kKQ8_0 or kKF16)
};

struct DecodeArgs {
    const uint8_t* region;   // slot 0 of the region holding the pages (resident or ring)
    int region_slot_base;    // global slot index of the region's first slot for the tensor map
    int region_slots;        // slots in the region (R or N)
    int slot0;               // region slot of unit 0
    int page0;               // absolute page index of unit 0
    int n_units;             // pages in this launch (consumed as 2 half-page stages each)
    int n_splits;            // splits of this launch; split s covers half-page stages
                             // [s*T/n_splits, (s+1)*T/n_splits) of the T = 2*n_units stages
    int split_base;          // first split index written by this launch
    int accumulate;          // tensor-core kernel: 1 = merge this launch's partials into the
                             // records already at split_base.. (the same stream's previous
                             // launch wrote them) instead of overwriting them
    int len;                 // tokens in the history
    int pos0, n_q;           // query positions pos0 .. pos0+n_q-1
    const __half* q;         // [n_q][n_qh][128]
    float q_scale;           // log2(e)/sqrt(128)
    int n_qh, n_kv, group;   // group = n_qh / n_kv
    int row_group_rows;      // rows handled per CTA (<= template ROWS)
    PartialBuffers part;
    int n_rows;              // n_q * n_qh
    int* err;                // device error word (bounded waits)
    int v_type;              // V type (kV*): with k_type, the page-head geometry
    int k_type;              // K type (kKQ8_0 or kKF16)
};

// query rows from which the merge writes out with 16-byte stores
constexpr int kMergeRowsMin = 1024;

struct MergeArgs {
    PartialBuffers part;
    int n_splits, n_rows;
    float* out;              // [n_rows][128]
    float* lse;              // [n_rows] or null
    const int* err;          // optional error word: when it is non-zero the
                             // merge writes NaN (a split's partial is missing)
};

// launchers (return cudaGetLastError())
cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                          cudaStream_t s);
// the same kernel reading the pages in place from mapped pinned host memory
// (a.region = the history's device alias) with 16-byte asynchronous copies
cudaError_t launch_decode_zero_copy(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                                    cudaStream_t s);
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s);
// multi-token (verify / prefill chunk) attention on tcgen05 tensor cores; same
// arguments and partial format as launch_decode
cudaError_t launch_chunk_mma(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                             cudaStream_t s);
// the same kernel reading the pages in place from mapped pinned host memory
cudaError_t launch_chunk_mma_zero_copy(const DecodeArgs& a, const CUtensorMap* kmap, int n_splits,
                                       cudaStream_t s);
size_t decode_smem_bytes();

// bounded-wait self-test kernel (one thread, an mbarrier nothing completes)
cudaError_t launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t s);
// copy `bytes` (a multiple of 16; both pointers 16-byte aligned) with plain
// 16-byte loads and stores, e.g. from a pinned host buffer's device alias
cudaError_t launch_copy16(void* dst, const void* src, size_t bytes, cudaStream_t s);

// record the calling thread's last error text (returned by kvs_last_error(NULL))
void set_last_error(const char* msg);

// error bits written to the device error word
enum : int {
    kErrWaitTimeout = 1,
};

}  // namespace kvs

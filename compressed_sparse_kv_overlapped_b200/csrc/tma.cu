// tma.cu -- host-side tensor-map encoding for the TMA loads (see tma.h).
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "tma.h"

namespace csa {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mu;

struct Entry {
    const void* base;
    uint64_t inner, rows, pitch;
    uint32_t box_inner, box_rows;
    bool swz;
    CUtensorMap map;
};
constexpr int kCache = 32;
Entry g_cache[kCache];
int g_used = 0, g_next = 0;

}  // namespace

cudaError_t tensor_map_2d_bf16(CUtensorMap* out, const void* base, uint64_t inner, uint64_t rows,
                               uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_used; ++i) {
        const Entry& e = g_cache[i];
        if (e.base == base && e.inner == inner && e.rows == rows && e.pitch == pitch_bytes &&
            e.box_inner == box_inner && e.box_rows == box_rows && e.swz == swizzle128) {
            *out = e.map;
            return cudaSuccess;
        }
    }
    if (!g_encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        cudaError_t err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (err != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    CUtensorMap m;
    std::memset(&m, 0, sizeof m);
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    Entry& e = g_cache[g_next];
    e = Entry{base, inner, rows, pitch_bytes, box_inner, box_rows, swizzle128, m};
    g_next = (g_next + 1) % kCache;
    if (g_used < kCache) ++g_used;
    *out = m;
    return cudaSuccess;
}

}  // namespace csa

// index_noalloc.cu -- csa_index_topk_noalloc: the indexer score + top-k call for callers that
// cannot hand the library a device workspace.
//
// Some callers have no way to obtain device memory at call time: code running under a framework
// whose caching allocator owns every device buffer and forbids direct cudaMalloc, real-time
// serving loops that must not allocate after start-up, or thin foreign-language bindings that see
// only the caller's input and output pointers.  For them this entry point keeps its scratch in a
// fixed array compiled into the library (kScratchBytes, about 14.2 MiB per device), so a call
// needs nothing but inputs, outputs and a stream.  The array occupies device memory on every GPU
// that loads the library until the process exits.
//
// The kernels are the same as those of csa_index_topk; only the scratch differs.
#include <mutex>

#include "kernels.h"

namespace csa {

namespace {

constexpr int kNoAllocMaxQ = 16;
constexpr int64_t kNoAllocMaxSlots = int64_t(1) << 20;  // Q * score-row stride
// Upper bound of index_ws_bytes(Q, e_stride) under the two limits above (each array rounded up to
// 256 bytes): histograms; fp32 scores; 64-bit kept-entry segments (each query's score
// row plus 128 entries); two words per scan chunk (chunks of at least 256 entries, nine more per
// query: a partial chunk and the ends of the final select's per-CTA prefixes); candidate keys (a
// quarter of the entries plus 256 per query).
constexpr size_t kScratchBytes = size_t(kNoAllocMaxQ) * kKeyBins * 4 + 256 +          // histograms, step words
                                 size_t(kNoAllocMaxSlots) * 4 + 256 +                  // scores
                                 size_t(kNoAllocMaxSlots + kNoAllocMaxQ * kSegPad) * 8 + 256 +
                                 2 * (size_t(kNoAllocMaxSlots / 256 + 9 * kNoAllocMaxQ) * 4 + 256) +
                                 size_t(kNoAllocMaxSlots / 4 + kNoAllocMaxQ * 256) * 8 + 256;

__device__ __align__(256) unsigned char g_index_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_dev[64] = {nullptr};

// Device address of g_index_scratch on the current device, looked up once per device.  (The name
// g_index_scratch in host code is a host-side stand-in, not a device address.)
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_dev[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_index_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = p;
    }
    *out = g_scratch_dev[dev];
    return cudaSuccess;
}

}  // namespace

}  // namespace csa

using namespace csa;

extern "C" int csa_index_topk_noalloc(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q,
                                      int64_t max_len, const csa_bf16* q_idx, const float* w,
                                      const csa_bf16* entry_keys, int32_t* idx_out, float* score_out,
                                      csa_stream_t stream) {
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q_idx || !w || !entry_keys || !idx_out)
        return set_error(CSA_ERR_ARG, "csa_index_topk_noalloc: NULL pointer argument");
    if (Q < 1 || max_len < 1) return set_error(CSA_ERR_ARG, "csa_index_topk_noalloc: Q < 1 or max_len < 1");
    if ((reinterpret_cast<uintptr_t>(q_idx) & 15u) || (reinterpret_cast<uintptr_t>(entry_keys) & 15u))
        return set_error(CSA_ERR_ARG, "csa_index_topk_noalloc: q_idx / entry_keys must be 16-byte aligned");
    const int64_t max_e = max_len / dims->m;
    int64_t es = ((max_e + 3) / 4) * 4;
    if (es < 4) es = 4;
    if (Q > kNoAllocMaxQ || (int64_t)Q * es > kNoAllocMaxSlots || index_ws_bytes(Q, es) > kScratchBytes)
        return set_error(CSA_ERR_UNSUPPORTED,
                         "csa_index_topk_noalloc: Q = %d queries of up to %lld entries exceed the built-in scratch "
                         "(at most %d queries and %lld query-entries in total); use csa_index_topk with a workspace",
                         Q, (long long)max_e, kNoAllocMaxQ, (long long)kNoAllocMaxSlots);
    void* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "csa_index_topk_noalloc: scratch address: %s", cudaGetErrorString(e));
    IndexParams ip{};
    ip.seqs = seqs;
    ip.queries = queries;
    ip.Q = Q;
    ip.H_I = dims->H_I;
    ip.d_I = dims->d_I;
    ip.m = dims->m;
    ip.k = dims->k;
    ip.q_idx = q_idx;
    ip.w = w;
    ip.entry_keys = entry_keys;
    ip.max_entries = max_e;
    ip.idx_out = idx_out;
    ip.score_out = score_out;
    if ((rc = device_status(&ip.status)) != CSA_OK) return rc;
    index_ws_carve(ip, scratch, Q, es);
    // the histogram must start at zero; clear it in case an earlier call was cut short
    e = launch_index_topk(ip, max_e, stream, /*zero_ws=*/true);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "csa_index_topk_noalloc: launch: %s", cudaGetErrorString(e));
    return CSA_OK;
}

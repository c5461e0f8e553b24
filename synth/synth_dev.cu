/*
 * synth_dev.cu -- device (CUDA) fill routines of the seeded input generator
 * defined in synth.h, for filling multi-gigabyte inputs directly in HBM.
 * Built with --fmad=false so that every operation of the definition is
 * rounded exactly as written; the host build (synth_host.c) produces the same
 * bits, which a GPU test checks.
 *
 * Every routine takes device pointers, enqueues one kernel on `stream` and
 * returns 0, or a negative value on a bad argument or launch failure.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth.h"

namespace {

enum { KIND_BF16_NORMAL = 0, KIND_F32_NORMAL = 1, KIND_F32_UNIFORM = 2 };

__global__ void fill_kernel(int kind, uint64_t key, int64_t ncols, int64_t r0, int64_t c0, int64_t nc,
                            int64_t n, double scale, void* out) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
        int64_t r = r0 + e / nc;
        int64_t c = c0 + e % nc;
        uint64_t i = (uint64_t)(r * ncols + c);
        if (kind == KIND_BF16_NORMAL) {
            ((uint16_t*)out)[e] = synth_bf16(scale * synth_normal(key, i));
        } else if (kind == KIND_F32_NORMAL) {
            ((float*)out)[e] = synth_f32(scale * synth_normal(key, i));
        } else {
            ((float*)out)[e] = synth_f32(scale * synth_uniform(key, i));
        }
    }
}

int launch(int kind, uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1, int64_t c0,
           int64_t c1, double scale, void* out, cudaStream_t stream) {
    if (!out || ncols <= 0 || r1 < r0 || c1 < c0 || c0 < 0 || c1 > ncols || r0 < 0) return -1;
    int64_t nc = c1 - c0, n = (r1 - r0) * nc;
    if (n == 0) return 0;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    uint64_t key = synth_key(seed, (uint64_t)tensor, (uint64_t)seq);
    fill_kernel<<<(unsigned)blocks, 256, 0, stream>>>(kind, key, ncols, r0, c0, nc, n, scale, out);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

} // namespace

extern "C" {

int synth_dev_fill_bf16_normal(uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
                               int64_t c0, int64_t c1, double scale, uint16_t* out, cudaStream_t stream) {
    return launch(KIND_BF16_NORMAL, seed, tensor, seq, ncols, r0, r1, c0, c1, scale, out, stream);
}

int synth_dev_fill_f32_normal(uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
                              int64_t c0, int64_t c1, double scale, float* out, cudaStream_t stream) {
    return launch(KIND_F32_NORMAL, seed, tensor, seq, ncols, r0, r1, c0, c1, scale, out, stream);
}

int synth_dev_fill_f32_uniform(uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
                               int64_t c0, int64_t c1, double scale, float* out, cudaStream_t stream) {
    return launch(KIND_F32_UNIFORM, seed, tensor, seq, ncols, r0, r1, c0, c1, scale, out, stream);
}

} // extern "C"

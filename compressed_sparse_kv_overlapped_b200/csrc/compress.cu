// compress.cu -- a1/a2: the token-axis softmax compressor, full-pass kernel.
//
// "DeepSeek V4 comprimeix el context: aixi funcionen CSA i HCA", sections "DeepSeek comprimeix la
// dimensio temporal" (an entry is a softmax-weighted sum of the tokens it summarises, with a
// separate weight per channel) and "Finestres solapades per evitar fronteres artificials"
// (overlapping windows, weights recomputed per window); "Frontier Techniques: NTK RoPE, CSA+HCA,
// QAT, MTP", 2.1 (m = 4) and 2.2 (m' = 128).
//
// HBM-bound streaming: every thread owns 8 consecutive channels (one 16-byte vector) of one entry
// and runs an online softmax over the window in fp32 (compress_dev.cuh), so each token row is
// read with coalesced 16-byte loads and the overlapping CSA windows re-read their shared rows from
// L1/L2.
#include "compress_dev.cuh"
#include "kernels.h"

namespace csa {

namespace {

__global__ void __launch_bounds__(256) compress_kernel(CompressParams p) {
    const int b = blockIdx.y;
    const csa_seq sq = p.seqs[b];
    const int64_t e0 = p.ranges ? p.ranges[2 * b] : p.range_begin;
    const int64_t e1 = p.ranges ? p.ranges[2 * b + 1] : p.range_end;
    if (e0 < 0 || e1 < e0 || (int64_t)p.m * e1 > sq.len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const int tpe = p.d >> 3;                 // threads per entry
    const int epc = blockDim.x / tpe;         // entries per CTA pass
    const int sub = threadIdx.x / tpe;
    const int g = threadIdx.x - sub * tpe;    // channel group: channels [8g, 8g+8)
    const int64_t out_off = p.which ? sq.hca_off : sq.csa_off;
    for (int64_t j = e0 + (int64_t)blockIdx.x * epc + sub; j < e1; j += (int64_t)gridDim.x * epc) {
        compress_entry8(j, p.m, p.win, p.d, p.d_I, g * 8, p.x, p.logit, p.bias, p.idx_key, sq.tok_off,
                        p.entries + (out_off + j) * p.d,
                        p.entry_keys ? p.entry_keys + (out_off + j) * p.d_I : nullptr);
    }
}

}  // namespace

cudaError_t launch_compress(const CompressParams& p, int64_t max_entries, cudaStream_t stream) {
    const int tpe = p.d / 8;
    const int epc = 256 / tpe;
    int64_t gx = (max_entries + epc - 1) / epc;
    if (gx < 1) gx = 1;
    if (gx > 8192) gx = 8192;
    compress_kernel<<<dim3((unsigned)gx, (unsigned)p.B), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace csa

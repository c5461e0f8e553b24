// compress_dev.cuh -- the per-entry compressor arithmetic, shared by the full-pass compressor
// kernel and the decode append kernel.
//
// "DeepSeek V4 comprimeix el context: aixi funcionen CSA i HCA", sections "DeepSeek comprimeix la
// dimensio temporal" and "Finestres solapades per evitar fronteres artificials".  Entry j covers
// tokens [m*j - (win - m), m*j + m) clipped at 0; per channel c the weights are
// softmax_t(logit_t[c] + bias[t - start][c]) and the entry is sum_t w_t x_t[c]; the indexer key
// (channels < d_I) reuses the same weights on idx_key.
#pragma once

#include "common.cuh"

namespace csa {

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// Channels [c0, c0+8) of entry j of one sequence (token rows start at tok0), written as bf16 to
// out_row (+ c0) and, when key_row != nullptr, the indexer key channels to key_row (+ c0).
// An online softmax over the window in fp32.  Tokens are taken 4 at a time: the loads of a batch
// are all issued before its softmax updates, so a 128-token window costs 32 memory round trips.
__device__ __forceinline__ void compress_entry8(int64_t j, int m, int win, int d, int d_I, int c0,
                                                const uint16_t* x, const uint16_t* logit, const float* bias,
                                                const uint16_t* idx_key, int64_t tok0, uint16_t* out_row,
                                                uint16_t* key_row) {
    constexpr int kBatch = 4;
    const int64_t start = (int64_t)m * j - (win - m);
    const int64_t t0 = start < 0 ? 0 : start;
    const int64_t t1 = (int64_t)m * j + m;
    const bool want_key = key_row != nullptr && idx_key != nullptr && c0 < d_I;
    float mx[8], den[8], acc[8], acck[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { mx[i] = -INFINITY; den[i] = 0.f; acc[i] = 0.f; acck[i] = 0.f; }
    for (int64_t tb = t0; tb < t1; tb += kBatch) {
        uint4 lv[kBatch], xv[kBatch], kv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int64_t t = tb + u;
            if (t < t1) {
                const int64_t row = tok0 + t;
                // coherent (L2) loads: at decode the newest token's rows may have been written by
                // this same kernel just before (csa_decode_args.new_rows)
                lv[u] = __ldcg(reinterpret_cast<const uint4*>(logit + row * d + c0));
                xv[u] = __ldcg(reinterpret_cast<const uint4*>(x + row * d + c0));
                if (want_key) kv[u] = __ldcg(reinterpret_cast<const uint4*>(idx_key + row * d_I + c0));
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (tb + u >= t1) break;
            float z[8], xf[8], kf[8];
            unpack8(lv[u], z);
            unpack8(xv[u], xf);
            const float4* bp = reinterpret_cast<const float4*>(bias + (tb + u - start) * d + c0);
            const float4 b0v = __ldg(bp), b1v = __ldg(bp + 1);  // parameters: L1/L2 resident
            z[0] += b0v.x; z[1] += b0v.y; z[2] += b0v.z; z[3] += b0v.w;
            z[4] += b1v.x; z[5] += b1v.y; z[6] += b1v.z; z[7] += b1v.w;
            if (want_key) unpack8(kv[u], kf);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (z[i] > mx[i]) {
                    const float r = expf(mx[i] - z[i]);  // 0 on the first token (mx = -inf)
                    den[i] = den[i] * r + 1.f;
                    acc[i] = acc[i] * r + xf[i];
                    if (want_key) acck[i] = acck[i] * r + kf[i];
                    mx[i] = z[i];
                } else {
                    const float e = expf(z[i] - mx[i]);
                    den[i] += e;
                    acc[i] = fmaf(e, xf[i], acc[i]);
                    if (want_key) acck[i] = fmaf(e, kf[i], acck[i]);
                }
            }
        }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0] / den[0], acc[1] / den[1]);
    o.y = pack_bf16x2(acc[2] / den[2], acc[3] / den[3]);
    o.z = pack_bf16x2(acc[4] / den[4], acc[5] / den[5]);
    o.w = pack_bf16x2(acc[6] / den[6], acc[7] / den[7]);
    *reinterpret_cast<uint4*>(out_row + c0) = o;
    if (want_key) {
        uint4 k;
        k.x = pack_bf16x2(acck[0] / den[0], acck[1] / den[1]);
        k.y = pack_bf16x2(acck[2] / den[2], acck[3] / den[3]);
        k.z = pack_bf16x2(acck[4] / den[4], acck[5] / den[5]);
        k.w = pack_bf16x2(acck[6] / den[6], acck[7] / den[7]);
        *reinterpret_cast<uint4*>(key_row + c0) = k;
    }
}

}  // namespace csa

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

// The softmax runs in base 2: a logit z (plus its bias) enters as z * log2(e), and every weight is
// 2^(difference) from the hardware exp2 approximation (relative error about 2^-22, far below the
// bf16 rounding of the entries), one subtraction and one special-function op per weight.  Maxima
// (M) are kept in the same base-2 scale.
constexpr float kLog2e = 1.4426950408889634f;

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
#pragma unroll
            for (int i = 0; i < 8; ++i) z[i] *= kLog2e;
            if (want_key) unpack8(kv[u], kf);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (z[i] > mx[i]) {
                    const float r = fast_exp2(mx[i] - z[i]);  // 0 on the first token (mx = -inf)
                    den[i] = den[i] * r + 1.f;
                    acc[i] = acc[i] * r + xf[i];
                    if (want_key) acck[i] = acck[i] * r + kf[i];
                    mx[i] = z[i];
                } else {
                    const float e = fast_exp2(z[i] - mx[i]);
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


// ---------------------------------------------------------------------------------------------
// Block-partial form (CSA ratio m = 4, HCA ratio m' a power of two from 4 to 128).  Per channel
// the softmax over a window is built from 4-token partials (z = logit + bias, M = max of the
// block's z in the base-2 scale, den = sum 2^(z log2(e) - M), acc = the same weights times x),
// merged pairwise:
//   CSA entry j = merge(P(tokens 4j-4..4j-1, bias rows 0..3), P(tokens 4j..4j+3, bias rows 4..7)),
//                 entry 0 = P(tokens 0..3, bias rows 4..7) alone (its window is clipped at 0);
//   HCA entry h = the balanced binary merge tree over its m'/4 blocks, in block order.
// Every step uses explicitly rounded fp32 operations (no contraction the compiler may choose
// differently in another kernel), and a merge is symmetric in its operands, so the full-pass kernel
// and the decode append produce bit-identical entries.
// ---------------------------------------------------------------------------------------------
struct Part8 {
    float M[8], den[8], acc[8], acck[8];
};

// Partial of 4 tokens: lg / xv / kv the tokens' logit / latent / indexer-key vectors (channels
// c0..c0+7), brow the 4 bias rows (fp32, channels c0..c0+7, row stride d).  valid[t] = false drops a
// token.  With KEYS the indexer key is accumulated with the same weights.
template <bool KEYS>
__device__ __forceinline__ void part4(const uint4 (&lg)[4], const uint4 (&xv)[4], const uint4 (&kv)[4],
                                      const float* brow, int d, Part8& P) {
    float z[4][8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float f[8];
        unpack8(lg[t], f);
        const float4 b0 = __ldg(reinterpret_cast<const float4*>(brow + t * d));
        const float4 b1 = __ldg(reinterpret_cast<const float4*>(brow + t * d) + 1);
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) z[t][i] = __fadd_rn(f[i], b[i]);
    }
    // M in the base-2 scale; a weight is 2^(z log2(e) - M), one fused multiply-add and one exp2
    float nM[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        P.M[i] = __fmul_rn(fmaxf(fmaxf(z[0][i], z[1][i]), fmaxf(z[2][i], z[3][i])), kLog2e);
        nM[i] = -P.M[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) { P.den[i] = 0.f; P.acc[i] = 0.f; P.acck[i] = 0.f; }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float xf[8], kf[8];
        unpack8(xv[t], xf);
        if (KEYS) unpack8(kv[t], kf);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float e = fast_exp2(__fmaf_rn(z[t][i], kLog2e, nM[i]));
            P.den[i] = __fadd_rn(P.den[i], e);
            P.acc[i] = __fmaf_rn(e, xf[i], P.acc[i]);
            if (KEYS) P.acck[i] = __fmaf_rn(e, kf[i], P.acck[i]);
        }
    }
}

// A <- merge(A, B); symmetric in A and B bit for bit.
template <bool KEYS>
__device__ __forceinline__ void merge8(Part8& A, const Part8& B) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float M = fmaxf(A.M[i], B.M[i]);
        const float fa = fast_exp2(__fsub_rn(A.M[i], M));
        const float fb = fast_exp2(__fsub_rn(B.M[i], M));
        A.den[i] = __fadd_rn(__fmul_rn(fa, A.den[i]), __fmul_rn(fb, B.den[i]));
        A.acc[i] = __fadd_rn(__fmul_rn(fa, A.acc[i]), __fmul_rn(fb, B.acc[i]));
        if (KEYS) A.acck[i] = __fadd_rn(__fmul_rn(fa, A.acck[i]), __fmul_rn(fb, B.acck[i]));
        A.M[i] = M;
    }
}

// acc / den.  den lies in [1, window] (the largest weight of a window is 2^0), so the fast
// reciprocal-based division is safe; its error (about 2 ulp in fp32) is far below the bf16
// rounding of the entries.
__device__ __forceinline__ float entry_div(float acc, float den) { return __fdividef(acc, den); }

// acc / den, rounded to bf16 (and the key accumulator with KEYS).
__device__ __forceinline__ uint4 finish8(const float (&acc)[8], const float (&den)[8]) {
    uint4 o;
    o.x = pack_bf16x2(entry_div(acc[0], den[0]), entry_div(acc[1], den[1]));
    o.y = pack_bf16x2(entry_div(acc[2], den[2]), entry_div(acc[3], den[3]));
    o.z = pack_bf16x2(entry_div(acc[4], den[4]), entry_div(acc[5], den[5]));
    o.w = pack_bf16x2(entry_div(acc[6], den[6]), entry_div(acc[7], den[7]));
    return o;
}

// Shuffle a partial from lane (lane ^ mask).
__device__ __forceinline__ void shfl_xor8(const Part8& A, Part8& B, int mask) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        B.M[i] = __shfl_xor_sync(0xffffffffu, A.M[i], mask);
        B.den[i] = __shfl_xor_sync(0xffffffffu, A.den[i], mask);
        B.acc[i] = __shfl_xor_sync(0xffffffffu, A.acc[i], mask);
    }
}

// CSA entry j (channels c0..c0+7) from the 8 rows of its window, rows fetched by fetch(tensor, t)
// for window position t in 0..7 (tensor 0: logit, 1: latent, 2: indexer key).  j = 0 uses positions
// 4..7 only.  val gets the entry's fp32 values (acc / den, rounded once); with KEYS, *key gets the
// indexer key as bf16.
template <bool KEYS, typename Fetch>
__device__ __forceinline__ void csa_entry_block4(int64_t j, int d, const float* bias_c0, Fetch fetch, float (&val)[8],
                                                 uint4* key) {
    uint4 lg[4], xv[4], kv[4];
    Part8 cur;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        lg[t] = fetch(0, 4 + t);
        xv[t] = fetch(1, 4 + t);
        kv[t] = KEYS ? fetch(2, 4 + t) : make_uint4(0, 0, 0, 0);
    }
    part4<KEYS>(lg, xv, kv, bias_c0 + 4 * d, d, cur);
    if (j > 0) {
        Part8 prev;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            lg[t] = fetch(0, t);
            xv[t] = fetch(1, t);
            kv[t] = KEYS ? fetch(2, t) : make_uint4(0, 0, 0, 0);
        }
        part4<KEYS>(lg, xv, kv, bias_c0, d, prev);
        merge8<KEYS>(cur, prev);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) val[i] = entry_div(cur.acc[i], cur.den[i]);
    if (KEYS) *key = finish8(cur.acck, cur.den);
}

// ---------------------------------------------------------------------------------------------
// Optional RMS normalization of every compressed entry ("DeepSeek V4 comprimeix el context",
// "CSA: buscar primer i atendre despres", last paragraph): out[c] = v[c] / sqrt(mean v^2 + eps) *
// gain[c].  An entry's channels are spread over 8 lanes (8 channels each) of each of the d/64 CTAs
// of a thread-block cluster; the sum of squares is added in a fixed order (each lane's 8 channels in
// order, a butterfly over the 8 lanes, the CTAs by rank) by both the full pass and the append.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float sumsq8(const float (&v)[8]) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s = __fmaf_rn(v[i], v[i], s);
    return s;
}

// Sum over the 8 lanes of an aligned lane group (every lane of the warp takes part; each group of 8
// ends with the same bits in all its lanes).
__device__ __forceinline__ float sum_lane8(float s) {
    s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 1));
    s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 2));
    s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 4));
    return s;
}

__device__ __forceinline__ float rms_inv(float ss, int d, float eps) {
    return __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)d), eps)));
}

// 8 entry values to bf16, normalized by inv * gain[c0 .. c0+7] when gain is given.
__device__ __forceinline__ uint4 entry_bf16(const float (&v)[8], const float* gain_c0, float inv) {
    float o[8];
    if (gain_c0) {
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(gain_c0));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(gain_c0) + 1);
        const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = __fmul_rn(__fmul_rn(v[i], inv), g[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = v[i];
    }
    uint4 r;
    r.x = pack_bf16x2(o[0], o[1]);
    r.y = pack_bf16x2(o[2], o[3]);
    r.z = pack_bf16x2(o[4], o[5]);
    r.w = pack_bf16x2(o[6], o[7]);
    return r;
}

// The total over the cluster's n CTAs of the value each holds at `p` (same offset in every CTA), in
// rank order.
__device__ __forceinline__ float cluster_sum(const float* p, int n) {
    float v[8];  // at most 8 slices (d <= 512); every load is issued before the sum
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = r < n ? ld_cluster_f32(p, (uint32_t)r) : 0.f;
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r)
        if (r < n) s = __fadd_rn(s, v[r]);
    return s;
}

// HCA entries of one 128-token tile, channels c0..c0+7: thread (u = tid / 8, g = tid % 8) of a
// 256-thread CTA holds the partial of tile block u (tokens 4u..4u+3) in P; the blocks of each entry
// (nb = m'/4 of them, a power of two up to 32) are merged by the binary tree in block order: lane
// shuffles for the two levels inside a warp (4 blocks per warp: u ^ 1 is lane ^ 8, u ^ 2 is
// lane ^ 16), then shared memory `xs` ([8 warps][8 g][24 floats]) for the levels across warps, one
// level per barrier.  Every thread of the CTA must call it (it contains barriers when nb >= 8).  On
// return lanes 0..7 of the first warp of each entry hold the merged partial in P.
__device__ __forceinline__ void hca_tree(Part8& P, int nb, float* xs) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    Part8 Q;
    if (nb >= 2) { shfl_xor8(P, Q, 8); merge8<false>(P, Q); }
    if (nb >= 4) { shfl_xor8(P, Q, 16); merge8<false>(P, Q); }
    if (nb < 8) return;
    const int wpe = nb / 4;  // warps per entry: 2, 4 or 8
    float* mine = xs + (warp * 8 + (lane & 7)) * 24;
    if (lane < 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) { mine[i] = P.M[i]; mine[8 + i] = P.den[i]; mine[16 + i] = P.acc[i]; }
    }
    for (int step = 1; step < wpe; step *= 2) {
        __syncthreads();
        if (lane < 8 && (warp & (2 * step - 1)) == 0) {
            const float* other = xs + ((warp + step) * 8 + lane) * 24;
#pragma unroll
            for (int i = 0; i < 8; ++i) { Q.M[i] = other[i]; Q.den[i] = other[8 + i]; Q.acc[i] = other[16 + i]; }
            merge8<false>(P, Q);
#pragma unroll
            for (int i = 0; i < 8; ++i) { mine[i] = P.M[i]; mine[8 + i] = P.den[i]; mine[16 + i] = P.acc[i]; }
        }
    }
}


// ---------------------------------------------------------------------------------------------
// HCA entries for m' a power of two from 16 to 128: warp w of the 256-thread CTA takes 16
// consecutive tokens of the entry (tokens 16w .. 16w+15 of a tile, or of the entry at decode), lane l
// the channel pair (2l, 2l+1) of the CTA's 64-channel slice.  Each lane forms the 16-token partial of
// its two channels; the m'/16 partials of an entry are merged in shared memory in a fixed balanced
// tree (warp order), with the same explicitly rounded steps as the 4-token form, so the full pass and
// the decode append produce identical entries.
// ---------------------------------------------------------------------------------------------
struct Part2 {
    float M[2], den[2], acc[2];
};

// Partial of 16 tokens: fetch(0, t) / fetch(1, t) give token t's logit / latent pair (two bf16 in a
// word, the even channel low), bias2(t) its bias row's pair.
template <typename Fetch, typename Bias>
__device__ __forceinline__ void hca_part16(Fetch fetch, Bias bias2, Part2& P) {
    float z[16][2];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const uint32_t l = fetch(0, t);
        const float2 b = bias2(t);
        z[t][0] = __fadd_rn(bf16lo(l), b.x);
        z[t][1] = __fadd_rn(bf16hi(l), b.y);
        mx0 = fmaxf(mx0, z[t][0]);
        mx1 = fmaxf(mx1, z[t][1]);
    }
    P.M[0] = __fmul_rn(mx0, kLog2e);
    P.M[1] = __fmul_rn(mx1, kLog2e);
    const float n0 = -P.M[0], n1 = -P.M[1];
    float d0 = 0.f, d1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const uint32_t x = fetch(1, t);
        const float e0 = fast_exp2(__fmaf_rn(z[t][0], kLog2e, n0));
        const float e1 = fast_exp2(__fmaf_rn(z[t][1], kLog2e, n1));
        d0 = __fadd_rn(d0, e0);
        d1 = __fadd_rn(d1, e1);
        a0 = __fmaf_rn(e0, bf16lo(x), a0);
        a1 = __fmaf_rn(e1, bf16hi(x), a1);
    }
    P.den[0] = d0;
    P.den[1] = d1;
    P.acc[0] = a0;
    P.acc[1] = a1;
}

// A <- merge(A, B); symmetric in A and B bit for bit (as merge8).
__device__ __forceinline__ void merge2(Part2& A, const Part2& B) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float M = fmaxf(A.M[i], B.M[i]);
        const float fa = fast_exp2(__fsub_rn(A.M[i], M));
        const float fb = fast_exp2(__fsub_rn(B.M[i], M));
        A.den[i] = __fadd_rn(__fmul_rn(fa, A.den[i]), __fmul_rn(fb, B.den[i]));
        A.acc[i] = __fadd_rn(__fmul_rn(fa, A.acc[i]), __fmul_rn(fb, B.acc[i]));
        A.M[i] = M;
    }
}

// Merge the partials of the wpe (1, 2, 4 or 8) consecutive warps of each entry: every warp stores
// its partial in xs ([8 warps][32 lanes][6 floats]), one barrier, then the first warp of each entry
// merges them pairwise by levels (warps 2i and 2i+1, then the pairs, ...).  Every thread of the CTA
// must call it when wpe > 1.  On return the first warp of each entry holds the merged partial in P.
__device__ __forceinline__ void hca_merge_warps(Part2& P, int wpe, float* xs) {
    if (wpe <= 1) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* mine = xs + (warp * 32 + lane) * 6;
    mine[0] = P.M[0]; mine[1] = P.M[1]; mine[2] = P.den[0]; mine[3] = P.den[1]; mine[4] = P.acc[0]; mine[5] = P.acc[1];
    __syncthreads();
    if (warp % wpe == 0) {
        Part2 L[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < wpe) {
                const float* o = xs + ((warp + k) * 32 + lane) * 6;
                L[k].M[0] = o[0]; L[k].M[1] = o[1]; L[k].den[0] = o[2]; L[k].den[1] = o[3];
                L[k].acc[0] = o[4]; L[k].acc[1] = o[5];
            }
        }
#pragma unroll
        for (int step = 1; step < 8; step *= 2)
#pragma unroll
            for (int k = 0; k < 8; k += 2 * step)
                if (step < wpe && k + step < wpe) merge2(L[k], L[k + step]);
        P = L[0];
    }
}

// Sum over the 32 lanes of a warp (every lane ends with the same bits).
__device__ __forceinline__ float warp_sum(float s) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
    return s;
}

// Two entry values to a bf16 pair, normalized by inv * gain[c], gain[c + 1] when gain is given (the
// same rounding steps as entry_bf16).
__device__ __forceinline__ uint32_t entry_bf16x2(float v0, float v1, const float* gain_c, float inv) {
    if (gain_c) {
        const float2 g = __ldg(reinterpret_cast<const float2*>(gain_c));
        v0 = __fmul_rn(__fmul_rn(v0, inv), g.x);
        v1 = __fmul_rn(__fmul_rn(v1, inv), g.y);
    }
    return pack_bf16x2(v0, v1);
}

}  // namespace csa

// attn.cu -- a5/a6/a7: MQA attention of all heads over a per-query key list on tcgen05 tensor
// cores, and the log-sum-exp merge of partial results.
//
// "DeepSeek V4 comprimeix el context: aixi funcionen CSA i HCA": one shared 512-wide latent is
// both key and value for every head ("DeepSeek comprimeix la dimensio temporal"); CSA attends the
// chosen compressed entries plus the local window ("CSA: buscar primer i atendre despres"); HCA
// attends every 128-token summary ("HCA: un resum global 128 vegades mes curt").  "Frontier
// Techniques: NTK RoPE, CSA+HCA, QAT, MTP", 2.1 (top-1024 + 128-token window) and 2.2.
//
// The key list of query i is [CSA slots idx[i][0..k) | raw window | HCA entries 0..floor(L/m')).
// It is cut into items of `keys_per_item` keys; one CTA computes one (query, item) pair:
//     S   = Q . K^T           (64 heads x 64 keys,  contraction over d)   tcgen05, M=64 N=64
//     P   = exp2(S*scale*log2e - m)  (online softmax, one row per thread)
//     O  += P . V             (64 heads x d, contraction over 64 keys)    tcgen05, M=64 N=256/128
// and writes either the final normalized output (single item) or a partial (O / l, lse) that
// combine_kernel merges by log-sum-exp.  The CSA/HCA merge of the method is exactly that merge.
//
// Layout: Q [64 x d] and each key tile [64 x d] live in shared memory as 128-byte-swizzled
// K-major blocks of 64 rows x 64 bf16; the key tile doubles as the MN-major B operand of the P.V
// product, so every key is loaded once.  TMEM holds S (64 columns) and O (d columns split over
// the two 16-lane halves of every sub-partition, the interleaved M=64 accumulator layout).
//
// Warp roles: warps 0-3 softmax + epilogue, warps 4-7 cp.async loaders (gathered rows, manual
// swizzle, zero-fill for masked slots), warp 8 TMEM allocator + single-thread MMA issuer.  Two
// key stages; every wait is bounded (kWaitLimitNs) and winds the CTA down on timeout.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kHeadsPad = 64;  // M of every MMA (heads beyond H are zero rows)
constexpr int kTileKeys = 64;
constexpr int kThreads = 288;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 256;

template <int D>
struct Smem {
    static constexpr int NKB = D / 64;                 // 64-wide blocks along d
    static constexpr int kBlock = 64 * 128;            // one block: 64 rows x 128 bytes
    static constexpr int kQ = 0;
    static constexpr int kK0 = kQ + NKB * kBlock;
    static constexpr int kK1 = kK0 + NKB * kBlock;
    static constexpr int kP = kK1 + NKB * kBlock;
    static constexpr int kBar = kP + kBlock;           // mbarriers
    static constexpr int kMisc = kBar + 16 * 8;        // tmem base, abort flag, masks
    static constexpr int kRowPtr = kMisc + 64;         // per loader warp: 16 row pointers
    static constexpr int kTotal = kRowPtr + 4 * 16 * 8;
    static constexpr int kAlloc = kTotal + 1024;       // slack for 1024-byte alignment
};

struct Bars {
    uint64_t full[2];   // loaders -> MMA / softmax: stage holds tile t
    uint64_t empty[2];  // MMA commit after P.V of the tile in the stage
    uint64_t s_full;    // MMA commit after Q.K^T
    uint64_t s_free;    // softmax finished reading S
    uint64_t p_full;    // softmax wrote P (and rescaled O)
    uint64_t o_done;    // MMA commit after P.V
    uint64_t fin;       // MMA commit before teardown
};

// Resolve slot `s` of query (qr, sq)'s key list [CSA slots | raw window | HCA entries] into a row
// pointer (nullptr = masked slot).
__device__ __forceinline__ const uint16_t* key_row(const AttnParams& p, int D, int qi, const csa_query& qr,
                                                   const csa_seq& sq, int64_t s) {
    if (s < p.k_slots) {
        const int32_t j = p.idx[(int64_t)qi * p.k_slots + s];
        if (j < 0) return nullptr;
        if ((int64_t)j >= qr.len / p.m) {
            report(p.status, CSA_ERR_INDEX);
            return nullptr;
        }
        return p.entries + (sq.csa_off + j) * D;
    }
    s -= p.k_slots;
    if (s < p.W) {
        const int64_t nw = qr.len < p.W ? qr.len : p.W;
        if (s >= nw) return nullptr;
        return p.raw + (sq.tok_off + qr.len - nw + s) * D;
    }
    s -= p.W;
    if (p.use_hca && s < qr.len / p.m_hca) return p.hca + (sq.hca_off + s) * D;
    return nullptr;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(AttnParams p) {
    using L = Smem<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Bars* bars = reinterpret_cast<Bars*>(sm + L::kBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::kMisc);  // [0] tmem base, [1] abort, [2..9] masks
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    uint16_t* mask16 = reinterpret_cast<uint16_t*>(misc + 2);     // [stage][4 warps]
    const uint32_t sbase = smem_u32(sm);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qi = blockIdx.y, item = blockIdx.x;
    const csa_query qr = p.queries[qi];
    const csa_seq sq = p.seqs[qr.seq];
    const bool qvalid = qr.len >= 1 && qr.len <= sq.len;
    const int64_t n_keys = (int64_t)p.k_slots + p.W + ((p.use_hca && qvalid) ? qr.len / p.m_hca : 0);
    const int64_t s0 = (int64_t)item * p.keys_per_item;
    int64_t s1 = min(n_keys, s0 + p.keys_per_item);
    if (s1 < s0) s1 = s0;
    if (!qvalid) {
        if (threadIdx.x == 0 && item == 0) report(p.status, CSA_ERR_INDEX);
        s1 = s0;
    }
    // once any CTA has given up on a wait, later CTAs do no work (bounded total time on a fault)
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == CSA_ERR_TIMEOUT) s1 = s0;
    const int T = s1 > s0 ? (int)((s1 - s0 + kTileKeys - 1) / kTileKeys) : 0;
    const int n_items = p.n_items;
    const bool direct = n_items == 1;

    if (threadIdx.x == 0) {
        mbar_init(&bars->full[0], 128);
        mbar_init(&bars->full[1], 128);
        mbar_init(&bars->empty[0], 1);
        mbar_init(&bars->empty[1], 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 128);
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->fin, 1);
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == 8 && T > 0) {
        tmem_alloc(misc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ loaders
        const int lw = warp - 4;
        const uint64_t* rowptr = reinterpret_cast<const uint64_t*>(sm + L::kRowPtr) + lw * 16;
        uint64_t* rowptr_w = reinterpret_cast<uint64_t*>(sm + L::kRowPtr) + lw * 16;
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        for (int t = 0; t < T; ++t) {
            const int st = t & 1;
            if (t >= 2 && !mbar_wait(&bars->empty[st], ((t >> 1) - 1) & 1, p.status, abort_flag)) break;
            if (t == 0) {
                // Q: 64 (padded) heads, 16 per loader warp
                for (int e = lane; e < 16 * CPR; e += 32) {
                    const int h = lw * 16 + e / CPR, ch = e % CPR;
                    const bool ok = h < p.H;
                    const uint16_t* src = ok ? p.q + ((int64_t)qi * p.H + h) * D + ch * 8 : p.q;
                    const uint32_t dst = sbase + L::kQ + (ch >> 3) * L::kBlock + sw128_offset(h, ch & 7);
                    cp_async16(dst, src, ok ? 16u : 0u);
                }
            }
            const int64_t tb = s0 + (int64_t)t * kTileKeys;
            bool valid = false;
            if (lane < 16) {
                const int64_t s = tb + lw * 16 + lane;
                const uint16_t* r = s < s1 ? key_row(p, D, qi, qr, sq, s) : nullptr;
                rowptr_w[lane] = reinterpret_cast<uint64_t>(r);
                valid = r != nullptr;
            }
            const uint32_t vm = __ballot_sync(0xffffffffu, valid) & 0xFFFFu;
            __syncwarp();
            const uint32_t kbase = sbase + (st ? L::kK1 : L::kK0);
            for (int e = lane; e < 16 * CPR; e += 32) {
                const int r = e / CPR, ch = e % CPR;
                const uint16_t* row = reinterpret_cast<const uint16_t*>(rowptr[r]);
                const int key = lw * 16 + r;
                const uint32_t dst = kbase + (ch >> 3) * L::kBlock + sw128_offset(key, ch & 7);
                cp_async16(dst, row ? row + ch * 8 : p.q, row ? 16u : 0u);
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            if (lane == 0) mask16[st * 4 + lw] = (uint16_t)vm;
            __syncwarp();
            mbar_arrive(&bars->full[st]);
        }
        cp_async_wait_all();
    } else if (warp == 8) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && T > 0) {
            constexpr uint32_t id1 = idesc_bf16(64, 64, false, false);
            constexpr int N2 = D >= 256 ? 256 : D;
            constexpr uint32_t id2 = idesc_bf16(64, N2, false, true);
            const uint32_t tS = tmem + kColS;
            auto gemm1 = [&](int t) {
                const uint32_t kb0 = sbase + ((t & 1) ? L::kK1 : L::kK0);
#pragma unroll 1
                for (int kb = 0; kb < L::NKB; ++kb) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t a = sdesc_kmajor(sbase + L::kQ + kb * L::kBlock + ks * 32);
                        const uint64_t b = sdesc_kmajor(kb0 + kb * L::kBlock + ks * 32);
                        umma_bf16(tS, a, b, id1, (kb | ks) != 0);
                    }
                }
            };
            auto gemm2 = [&](int t) {
                const uint32_t kb0 = sbase + ((t & 1) ? L::kK1 : L::kK0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = sdesc_kmajor(sbase + L::kP + ks * 32);
#pragma unroll
                    for (int half = 0; half < (D >= 256 ? D / 256 : 1); ++half) {
                        // V rows ks*16 .. ks*16+15 of the key tile, dims [half*256, half*256 + N2)
                        const uint64_t b = sdesc_mnmajor(kb0 + half * 4 * L::kBlock + ks * 16 * 128, L::kBlock);
                        const uint32_t tO = tmem + kColO + ((uint32_t)(half * 16) << 16);
                        umma_bf16(tO, a, b, id2, (t > 0 || ks > 0) ? 1u : 0u);
                    }
                }
            };
            bool ok = mbar_wait(&bars->full[0], 0, p.status, abort_flag);
            if (ok) {
                tc_fence_after();
                gemm1(0);
                umma_commit(&bars->s_full);
            }
            for (int t = 0; ok && t < T; ++t) {
                if (t + 1 < T) {
                    ok = mbar_wait(&bars->full[(t + 1) & 1], ((t + 1) >> 1) & 1, p.status, abort_flag) &&
                         mbar_wait(&bars->s_free, t & 1, p.status, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    gemm1(t + 1);
                    umma_commit(&bars->s_full);
                }
                ok = mbar_wait(&bars->p_full, t & 1, p.status, abort_flag);
                if (!ok) break;
                tc_fence_after();
                gemm2(t);
                umma_commit(&bars->empty[t & 1]);
                umma_commit(&bars->o_done);
            }
            umma_commit(&bars->fin);
            mbar_wait(&bars->fin, 0, p.status, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax + epilogue
        const int i = lane;
        const bool row_thread = i < 16;
        const int h = warp * 16 + (i & 15);                 // head row handled by this lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int st = t & 1;
            ok = mbar_wait(&bars->s_full, t & 1, p.status, abort_flag) &&
                 mbar_wait(&bars->full[st], (t >> 1) & 1, p.status, abort_flag);
            if (!ok) break;
            tc_fence_after();
            float s[64];
            {
                uint32_t r[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    tmem_ld16(tmem + lane_base + kColS + q4 * 16, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) s[q4 * 16 + j] = __uint_as_float(r[j]);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->s_free);
            const uint64_t vmask = (uint64_t)mask16[st * 4 + 0] | ((uint64_t)mask16[st * 4 + 1] << 16) |
                                   ((uint64_t)mask16[st * 4 + 2] << 32) | ((uint64_t)mask16[st * 4 + 3] << 48);
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                s[j] = ((vmask >> j) & 1ull) ? s[j] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[j]);
            }
            // lazy rescaling: move the reference max only when it grows by more than 2^8
            float alpha = 1.f;
            if (mx > m_run + 8.f) {
                alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - mx);
                m_run = mx;
                l_run *= alpha;
            }
            // P buffer and O are free once the previous P.V finished
            if (t > 0) {
                ok = mbar_wait(&bars->o_done, (t - 1) & 1, p.status, abort_flag);
                if (!ok) break;
                tc_fence_after();
                // rescale O rows whose reference max moved (warp-collective TMEM access)
                const float a_lo = __shfl_sync(0xffffffffu, alpha, i & 15);
                const float a_me = row_thread ? alpha : a_lo;
                const bool any = __any_sync(0xffffffffu, row_thread && alpha != 1.f);
                if (any) {
                    constexpr int OC = D >= 256 ? 256 : D;
#pragma unroll 1
                    for (int c = 0; c < OC; c += 16) {
                        uint32_t r[16];
                        tmem_ld16(tmem + lane_base + kColO + c, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a_me);
                        tmem_st16(tmem + lane_base + kColO + c, r);
                    }
                    tmem_st_wait();
                }
            }
            if (row_thread) {
                float lsum = 0.f;
                unsigned char* prow = sm + L::kP;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float p0 = m_run == -INFINITY ? 0.f : exp2f(s[c8 * 8 + 2 * u] - m_run);
                        const float p1 = m_run == -INFINITY ? 0.f : exp2f(s[c8 * 8 + 2 * u + 1] - m_run);
                        w4[u] = pack_bf16x2(p0, p1);
                        lsum += bf16lo(w4[u]) + bf16hi(w4[u]);
                    }
                    *reinterpret_cast<uint4*>(prow + sw128_offset(h, c8)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                l_run += lsum;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full);
        }
        // ---- epilogue
        if (ok && T > 0) ok = mbar_wait(&bars->o_done, (T - 1) & 1, p.status, abort_flag);
        const float l_row = __shfl_sync(0xffffffffu, l_run, i & 15);
        const float m_row = __shfl_sync(0xffffffffu, m_run, i & 15);
        const bool has = ok && T > 0 && l_row > 0.f;
        const float inv = has ? 1.f / l_row : 0.f;
        constexpr int OC = D >= 256 ? 256 : D;
        const int dim0 = row_thread ? 0 : 256;
        const bool writes = (row_thread || D >= 512) && h < p.H;
        float* orow = direct ? p.out + ((int64_t)qi * p.H + h) * D
                             : p.part_o + (((int64_t)qi * n_items + item) * kHeadsPad + h) * D;
        if (has) tc_fence_after();
        if (has || direct) {
#pragma unroll 1
            for (int c = 0; c < OC; c += 16) {
                uint32_t r[16];
                if (has) {
                    tmem_ld16(tmem + lane_base + kColO + c, r);
                    tmem_ld_wait();
                }
                if (writes) {
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        float4 v;
                        v.x = has ? __uint_as_float(r[j]) * inv : 0.f;
                        v.y = has ? __uint_as_float(r[j + 1]) * inv : 0.f;
                        v.z = has ? __uint_as_float(r[j + 2]) * inv : 0.f;
                        v.w = has ? __uint_as_float(r[j + 3]) * inv : 0.f;
                        *reinterpret_cast<float4*>(orow + dim0 + c + j) = v;
                    }
                }
            }
        }
        if (row_thread && h < p.H) {
            const float lse_v = has ? (m_row + log2f(l_row)) * 0.69314718055994531f : -INFINITY;
            if (direct) {
                if (p.lse) p.lse[(int64_t)qi * p.H + h] = lse_v;
            } else {
                p.part_lse[((int64_t)qi * n_items + item) * kHeadsPad + h] = lse_v;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8 && T > 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// out[q][h] = sum_items exp(lse_i - lse) * O_i,  lse = logsumexp_i lse_i  (items with lse = -inf
// contribute nothing and are not read).
template <int D>
__global__ void combine_kernel(AttnParams p) {
    const int h = blockIdx.x, qi = blockIdx.y;
    const int n_items = p.n_items;
    __shared__ float wts[256];
    __shared__ float s_lse;
    if (threadIdx.x == 0) {
        float mx = -INFINITY;
        for (int it = 0; it < n_items; ++it)
            mx = fmaxf(mx, p.part_lse[((int64_t)qi * n_items + it) * kHeadsPad + h]);
        float sum = 0.f;
        for (int it = 0; it < n_items; ++it) {
            const float l = p.part_lse[((int64_t)qi * n_items + it) * kHeadsPad + h];
            const float w = mx == -INFINITY ? 0.f : expf(l - mx);
            wts[it] = w;
            sum += w;
        }
        const float lse = mx == -INFINITY ? -INFINITY : mx + logf(sum);
        for (int it = 0; it < n_items; ++it) wts[it] = sum > 0.f ? wts[it] / sum : 0.f;
        s_lse = lse;
        if (p.lse) p.lse[(int64_t)qi * p.H + h] = lse;
    }
    __syncthreads();
    for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int it = 0; it < n_items; ++it) {
            const float w = wts[it];
            if (w == 0.f) continue;
            const float4 v = *reinterpret_cast<const float4*>(
                p.part_o + (((int64_t)qi * n_items + it) * kHeadsPad + h) * D + c);
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(p.out + ((int64_t)qi * p.H + h) * D + c) = acc;
    }
}

template <int D>
cudaError_t launch_d(AttnParams& p, cudaStream_t stream) {
    using L = Smem<D>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const int n_items = p.n_items;
    attn_kernel<D><<<dim3((unsigned)n_items, (unsigned)p.Q), kThreads, L::kAlloc, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || n_items == 1) return e;
    combine_kernel<D><<<dim3((unsigned)p.H, (unsigned)p.Q), D / 4, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t attn_ws_bytes(int Q, int items, int d) {
    if (items <= 1) return 0;
    const size_t o = (size_t)Q * items * kHeadsPad * d * 4;
    const size_t l = (size_t)Q * items * kHeadsPad * 4;
    return ((o + 255) & ~(size_t)255) + ((l + 255) & ~(size_t)255);
}

cudaError_t launch_attention(AttnParams& p, void* ws, cudaStream_t stream) {
    const int n_items = p.n_items;
    if (n_items > 1) {
        const size_t o = (size_t)p.Q * n_items * kHeadsPad * p.d * 4;
        p.part_o = static_cast<float*>(ws);
        p.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + ((o + 255) & ~(size_t)255));
    }
    if (p.d == 512) return launch_d<512>(p, stream);
    if (p.d == 128) return launch_d<128>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace csa

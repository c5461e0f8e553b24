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
// It is cut into items (the front part and the HCA part separately, so the HCA items do not depend
// on the top-k and can run while it is computed); one CTA computes one (query, item) pair:
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
    static constexpr int kP0 = kK1 + NKB * kBlock;     // P, double-buffered
    static constexpr int kP1 = kP0 + kBlock;
    static constexpr int kBar = kP1 + kBlock;          // mbarriers
    static constexpr int kMisc = kBar + 16 * 8;        // tmem base, abort flag, masks
    static constexpr int kRowPtr = kMisc + 64;         // per loader warp: 16 row pointers
    static constexpr int kTotal = kRowPtr + 4 * 16 * 8;
    static constexpr int kAlloc = kTotal + 1024;       // slack for 1024-byte alignment
};

struct Bars {
    uint64_t full[2];    // loaders -> MMA / softmax: key stage holds tile t
    uint64_t empty[2];   // MMA commit after P.V of the tile in the stage
    uint64_t s_full;     // MMA commit after Q.K^T
    uint64_t s_free;     // softmax finished reading S
    uint64_t p_full[2];  // softmax wrote P buffer t&1 (and rescaled O if needed)
    uint64_t o_done[2];  // MMA commit after the P.V that read P buffer t&1
    uint64_t fin;        // MMA commit before teardown
};

// Per-CTA constants of the key list [CSA slots | raw window | HCA entries] of one query.
struct KeyList {
    const int32_t* idx;      // this query's k slots
    int64_t n_causal;        // floor(L / m)
    int64_t n_hca;           // floor(L / m') (0 without HCA)
    int64_t win_row0;        // raw row of the first window token
    int64_t nw;              // window tokens present
    int64_t csa_row0, hca_row0;
};

// Row pointer of slot `s` (nullptr = masked slot).
__device__ __forceinline__ const uint16_t* key_row(const AttnParams& p, int D, const KeyList& kl, int64_t s) {
    if (s < p.k_slots) {
        const int32_t j = kl.idx[s];
        if (j < 0) return nullptr;
        if ((int64_t)j >= kl.n_causal) {
            report(p.status, CSA_ERR_INDEX);
            return nullptr;
        }
        return p.entries + (kl.csa_row0 + j) * D;
    }
    s -= p.k_slots;
    if (s < p.W) return s < kl.nw ? p.raw + (kl.win_row0 + s) * D : nullptr;
    s -= p.W;
    return s < kl.n_hca ? p.hca + (kl.hca_row0 + s) * D : nullptr;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(AttnParams p, int p_item_base) {
    using L = Smem<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Bars* bars = reinterpret_cast<Bars*>(sm + L::kBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::kMisc);  // [0] tmem base, [1] abort, [2..5] masks
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    uint16_t* mask16 = reinterpret_cast<uint16_t*>(misc + 2);     // [stage][4 warps]
    const uint32_t sbase = smem_u32(sm);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qi = blockIdx.y, item = blockIdx.x + p_item_base;
    // The query table and sequence lengths come from kernels at least two launches back, which are
    // complete once this grid runs (every kernel of the chain waits before it lets the next start).
    const csa_query qr = p.queries[qi];
    const csa_seq sq = p.seqs[qr.seq];
    const bool qvalid = qr.len >= 1 && qr.len <= sq.len;
    KeyList kl;
    kl.idx = p.idx ? p.idx + (int64_t)qi * p.k_slots : nullptr;
    kl.n_causal = qr.len / p.m;
    kl.n_hca = (p.use_hca && qvalid) ? qr.len / p.m_hca : 0;
    kl.nw = qr.len < p.W ? qr.len : p.W;
    kl.win_row0 = sq.tok_off + qr.len - kl.nw;
    kl.csa_row0 = sq.csa_off;
    kl.hca_row0 = sq.hca_off;
    const int64_t front = (int64_t)p.k_slots + p.W;
    const int64_t n_keys = front + kl.n_hca;
    int64_t s0, s1;
    if (p.n_items == 1) {
        s0 = 0;
        s1 = n_keys;
    } else if (item < p.items_front) {
        s0 = (int64_t)item * p.kpi_front;
        s1 = min(front, s0 + p.kpi_front);
    } else {
        s0 = front + (int64_t)(item - p.items_front) * p.kpi_hca;
        s1 = min(n_keys, s0 + p.kpi_hca);
    }
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
    const bool dep_wait = !(p.hca_nowait && !direct && item >= p.items_front);

    if (threadIdx.x == 0) {
        mbar_init(&bars->full[0], 128);
        mbar_init(&bars->full[1], 128);
        mbar_init(&bars->empty[0], 1);
        mbar_init(&bars->empty[1], 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 128);
        mbar_init(&bars->p_full[0], 128);
        mbar_init(&bars->p_full[1], 128);
        mbar_init(&bars->o_done[0], 1);
        mbar_init(&bars->o_done[1], 1);
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
        // Lane l copies 16-byte chunks l, l+32, ... of each 64-chunk (1 KiB) row: chunk c lands in
        // block c/8 at swizzled position (c%8) ^ (row%8), and c%8 = l%8 for every chunk of a lane.
        constexpr int CPL = CPR / 32 > 0 ? CPR / 32 : 1;  // chunks per lane per row (2 at D = 512)
        const uint32_t lane_blk = (uint32_t)(lane >> 3) * L::kBlock;  // block of chunk `lane`
        const uint32_t lane_c7 = (uint32_t)(lane & 7);
        if (T > 0) {
            // Q: 64 (padded) heads, 16 per loader warp; an input, so it may load before the wait
            for (int r = 0; r < 16; ++r) {
                const int h = lw * 16 + r;
                const bool ok = h < p.H;
                const uint16_t* src = p.q + ((int64_t)qi * p.H + (ok ? h : 0)) * D;
                const uint32_t dst = sbase + L::kQ + lane_blk + (uint32_t)h * 128u + ((lane_c7 ^ (h & 7)) << 4);
                if (CPR >= 32) {
#pragma unroll
                    for (int u = 0; u < CPL; ++u)
                        cp_async16(dst + u * 4 * L::kBlock, src + (lane + 32 * u) * 8, ok ? 16u : 0u);
                } else if (lane < CPR) {
                    cp_async16(dst, src + lane * 8, ok ? 16u : 0u);
                }
            }
        }
        if (dep_wait) grid_dep_wait();  // the selected indices come from the previous kernel
        for (int t = 0; t < T; ++t) {
            const int st = t & 1;
            if (t >= 2 && !mbar_wait(&bars->empty[st], ((t >> 1) - 1) & 1, p.status, abort_flag)) break;
            const int64_t tb = s0 + (int64_t)t * kTileKeys;
            bool valid = false;
            if (lane < 16) {
                const int64_t s = tb + lw * 16 + lane;
                const uint16_t* r = s < s1 ? key_row(p, D, kl, s) : nullptr;
                rowptr_w[lane] = reinterpret_cast<uint64_t>(r);
                valid = r != nullptr;
            }
            const uint32_t vm = __ballot_sync(0xffffffffu, valid) & 0xFFFFu;
            __syncwarp();
            const uint32_t kbase = sbase + (st ? L::kK1 : L::kK0) + lane_blk;
#pragma unroll 4
            for (int r = 0; r < 16; ++r) {
                const uint16_t* row = reinterpret_cast<const uint16_t*>(rowptr[r]);
                const int key = lw * 16 + r;
                const uint32_t dst = kbase + (uint32_t)key * 128u + ((lane_c7 ^ (key & 7)) << 4);
                const uint32_t nb = row ? 16u : 0u;
                const uint16_t* src = row ? row : p.q;
                if (CPR >= 32) {
#pragma unroll
                    for (int u = 0; u < CPL; ++u) cp_async16(dst + u * 4 * L::kBlock, src + (lane + 32 * u) * 8, nb);
                } else if (lane < CPR) {
                    cp_async16(dst, src + lane * 8, nb);
                }
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
        if (dep_wait) grid_dep_wait();
        if (lane == 0 && T > 0) {
            constexpr uint32_t id1 = idesc_bf16(64, 64, false, false);
            constexpr int N2 = D >= 256 ? 256 : D;
            constexpr int HALVES = D >= 256 ? D / 256 : 1;
            constexpr uint32_t id2 = idesc_bf16(64, N2, false, true);
            const uint32_t tS = tmem + kColS;
            // descriptor bases; the start address field is (address >> 4) in the low bits
            const uint64_t dQ = sdesc_kmajor(sbase + L::kQ);
            const uint64_t dK[2] = {sdesc_kmajor(sbase + L::kK0), sdesc_kmajor(sbase + L::kK1)};
            const uint64_t dV[2] = {sdesc_mnmajor(sbase + L::kK0, L::kBlock), sdesc_mnmajor(sbase + L::kK1, L::kBlock)};
            const uint64_t dP[2] = {sdesc_kmajor(sbase + L::kP0), sdesc_kmajor(sbase + L::kP1)};
            auto gemm1 = [&](int t) {
                const uint64_t kd = dK[t & 1];
#pragma unroll 1
                for (int kb = 0; kb < L::NKB; ++kb) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t off = (uint64_t)((kb * L::kBlock + ks * 32) >> 4);
                        umma_bf16(tS, dQ + off, kd + off, id1, (kb | ks) != 0);
                    }
                }
            };
            auto gemm2 = [&](int t) {
                const uint64_t vd = dV[t & 1], pd = dP[t & 1];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                    for (int half = 0; half < HALVES; ++half) {
                        // V rows ks*16 .. ks*16+15 of the key tile, dims [half*256, half*256 + N2)
                        const uint64_t b = vd + (uint64_t)((half * 4 * L::kBlock + ks * 16 * 128) >> 4);
                        const uint32_t tO = tmem + kColO + ((uint32_t)(half * 16) << 16);
                        umma_bf16(tO, pd + (uint64_t)((ks * 32) >> 4), b, id2, (t > 0 || ks > 0) ? 1u : 0u);
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
                ok = mbar_wait(&bars->p_full[t & 1], (t >> 1) & 1, p.status, abort_flag);
                if (!ok) break;
                tc_fence_after();
                gemm2(t);
                umma_commit(&bars->empty[t & 1]);
                umma_commit(&bars->o_done[t & 1]);
            }
            umma_commit(&bars->fin);
            mbar_wait(&bars->fin, 0, p.status, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax + epilogue
        if (dep_wait) grid_dep_wait();
        grid_dep_launch();
        const int i = lane;
        const bool row_thread = i < 16;
        const int h = warp * 16 + (i & 15);                 // head row handled by this lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        constexpr int OC = D >= 256 ? 256 : D;              // O columns held by each lane
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
                uint32_t r[4][16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tmem + lane_base + kColS + q4 * 16, r[q4]);
                tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                    for (int j = 0; j < 16; ++j) s[q4 * 16 + j] = __uint_as_float(r[q4][j]);
            }
            tc_fence_before();
            mbar_arrive(&bars->s_free);
            const uint64_t vmask = (uint64_t)mask16[st * 4 + 0] | ((uint64_t)mask16[st * 4 + 1] << 16) |
                                   ((uint64_t)mask16[st * 4 + 2] << 32) | ((uint64_t)mask16[st * 4 + 3] << 48);
            float mx = -INFINITY;
            const float sc = p.scale_log2;
            if (vmask == ~0ull) {
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    s[j] *= sc;
                    mx = fmaxf(mx, s[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    s[j] = ((vmask >> j) & 1ull) ? s[j] * sc : -INFINITY;
                    mx = fmaxf(mx, s[j]);
                }
            }
            // lazy rescaling: move the reference max only when it grows by more than 2^8
            float alpha = 1.f;
            if (mx > m_run + 8.f) {
                alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - mx);
                m_run = mx;
                l_run *= alpha;
            }
            // O must hold every earlier P.V before it is rescaled (rare)
            const bool any = __any_sync(0xffffffffu, row_thread && alpha != 1.f);
            if (t > 0 && any) {
                ok = mbar_wait(&bars->o_done[(t - 1) & 1], ((t - 1) >> 1) & 1, p.status, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const float a_me = __shfl_sync(0xffffffffu, alpha, i & 15);
#pragma unroll 1
                for (int c = 0; c < OC; c += 64) {
                    uint32_t r[4][16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tmem + lane_base + kColO + c + q4 * 16, r[q4]);
                    tmem_ld_wait();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) r[q4][j] = __float_as_uint(__uint_as_float(r[q4][j]) * a_me);
                        tmem_st16(tmem + lane_base + kColO + c + q4 * 16, r[q4]);
                    }
                }
                tmem_st_wait();
            }
            // P buffer t&1 is free once the P.V of tile t-2 finished
            if (t >= 2) {
                ok = mbar_wait(&bars->o_done[st], ((t >> 1) - 1) & 1, p.status, abort_flag);
                if (!ok) break;
            }
            if (row_thread) {
                // masked slots hold -inf: 2^(-inf - m) = 0; while the row has seen no key, m_use = 0
                const float m_use = m_run == -INFINITY ? 0.f : m_run;
                float lsum = 0.f;
                const uint32_t prow = sbase + (st ? L::kP1 : L::kP0);
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float p0 = fast_exp2(s[c8 * 8 + 2 * u] - m_use);
                        const float p1 = fast_exp2(s[c8 * 8 + 2 * u + 1] - m_use);
                        lsum += p0 + p1;
                        w4[u] = pack_bf16x2(p0, p1);
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + sw128_offset(h, c8)),
                                 "r"(w4[0]), "r"(w4[1]), "r"(w4[2]), "r"(w4[3])
                                 : "memory");
                }
                l_run += lsum;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full[st]);
        }
        // ---- epilogue: TMEM -> shared memory (Q and the key stages are free now) -> coalesced stores
        if (ok && T > 0) ok = mbar_wait(&bars->o_done[(T - 1) & 1], ((T - 1) >> 1) & 1, p.status, abort_flag);
        const float l_row = __shfl_sync(0xffffffffu, l_run, i & 15);
        const float m_row = __shfl_sync(0xffffffffu, m_run, i & 15);
        const bool has = ok && T > 0 && l_row > 0.f;
        const float inv = has ? 1.f / l_row : 0.f;
        const int dim0 = row_thread ? 0 : 256;
        const bool mine = row_thread || D >= 512;  // lanes 16-31 hold dims 256-511 when D = 512
        // staging rows of D floats, padded by 4 floats so 16-byte row-strided writes spread banks
        constexpr int kStride = D + 4;
        float* stage = reinterpret_cast<float*>(sm + L::kQ);  // Q and both key stages are free now
        static_assert(64 * (D + 4) * 4 <= 3 * L::NKB * L::kBlock, "epilogue staging exceeds Q + key stages");
        if (has) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < OC; c += 64) {
                uint32_t r[4][16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tmem + lane_base + kColO + c + q4 * 16, r[q4]);
                tmem_ld_wait();
                if (mine) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                        for (int j = 0; j < 16; j += 4) {
                            float4 v;
                            v.x = __uint_as_float(r[q4][j]) * inv;
                            v.y = __uint_as_float(r[q4][j + 1]) * inv;
                            v.z = __uint_as_float(r[q4][j + 2]) * inv;
                            v.w = __uint_as_float(r[q4][j + 3]) * inv;
                            *reinterpret_cast<float4*>(stage + h * kStride + dim0 + c + q4 * 16 + j) = v;
                        }
                }
            }
        }
        // staged rows become visible to the bulk-copy engine (async proxy) after this fence + barrier
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the four softmax warps (128 threads)
        const int rows = p.H < kHeadsPad ? p.H : kHeadsPad;
        if (has) {
            // one lane per warp hands 16 staged rows to the bulk-copy engine
            if (i == 0) {
                for (int hh = warp * 16; hh < warp * 16 + 16 && hh < rows; ++hh) {
                    float* dst = direct ? p.out + ((int64_t)qi * p.H + hh) * D
                                        : p.part_o + (((int64_t)qi * n_items + item) * kHeadsPad + hh) * D;
                    bulk_store(dst, smem_u32(stage + hh * kStride), D * 4);
                }
                bulk_commit();
                bulk_wait_all();
            }
        } else if (direct) {
            const int tid = threadIdx.x;  // 0..127
            for (int e = tid; e < rows * (D / 4); e += 128) {
                const int hh = e / (D / 4), c4 = e % (D / 4);
                *reinterpret_cast<float4*>(p.out + ((int64_t)qi * p.H + hh) * D + c4 * 4) =
                    make_float4(0.f, 0.f, 0.f, 0.f);
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
// contribute nothing and are not read).  One CTA per (head, query); warp 0 computes the weights, then
// every thread accumulates one float4 column of all contributing partials with batched loads.
template <int D>
__global__ void combine_kernel(AttnParams p) {
    constexpr int kMaxBatch = 24;  // partial rows held in registers per pass
    grid_dep_wait();  // the partials come from the attention grid
    const int h = blockIdx.x, qi = blockIdx.y;
    const int n_items = p.n_items;
    const int lane = threadIdx.x & 31;
    __shared__ float s_lse[256];
    __shared__ float s_w[256];
    __shared__ float s_res[2];
    // every thread owns one float4 column of the output row (D/4 threads)
    const int c = threadIdx.x * 4;
    const float* base = p.part_o + ((int64_t)qi * n_items * kHeadsPad + h) * D + c;
    const int64_t item_stride = (int64_t)kHeadsPad * D;
    for (int it = threadIdx.x; it < n_items; it += blockDim.x)
        s_lse[it] = __ldcg(p.part_lse + ((int64_t)qi * n_items + it) * kHeadsPad + h);
    // the partial rows do not depend on the weights: issue their loads first
    float4 v[kMaxBatch];
    const int nb0 = n_items < kMaxBatch ? n_items : kMaxBatch;
#pragma unroll
    for (int u = 0; u < kMaxBatch; ++u)
        if (u < nb0) v[u] = __ldcg(reinterpret_cast<const float4*>(base + u * item_stride));
    __syncthreads();
    if (threadIdx.x < 32) {
        float mx = -INFINITY;
        for (int it = lane; it < n_items; it += 32) mx = fmaxf(mx, s_lse[it]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int it = lane; it < n_items; it += 32) {
            const float w = mx == -INFINITY ? 0.f : expf(s_lse[it] - mx);
            s_w[it] = w;
            sum += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            s_res[0] = sum > 0.f ? 1.f / sum : 0.f;
            s_res[1] = mx == -INFINITY ? -INFINITY : mx + logf(sum);
        }
    }
    __syncthreads();
    const float inv = s_res[0];
    if (threadIdx.x == 0 && p.lse) p.lse[(int64_t)qi * p.H + h] = s_res[1];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int b = 0; b < n_items; b += kMaxBatch) {
        const int nb = n_items - b < kMaxBatch ? n_items - b : kMaxBatch;
        if (b > 0) {
#pragma unroll
            for (int u = 0; u < kMaxBatch; ++u)
                if (u < nb) v[u] = __ldcg(reinterpret_cast<const float4*>(base + (b + u) * item_stride));
        }
#pragma unroll
        for (int u = 0; u < kMaxBatch; ++u) {
            if (u < nb) {
                const float w = s_w[b + u] * inv;
                if (w > 0.f) {  // an empty item (lse = -inf) has weight 0 and unwritten rows
                    acc.x = fmaf(w, v[u].x, acc.x);
                    acc.y = fmaf(w, v[u].y, acc.y);
                    acc.z = fmaf(w, v[u].z, acc.z);
                    acc.w = fmaf(w, v[u].w, acc.w);
                }
            }
        }
    }
    *reinterpret_cast<float4*>(p.out + ((int64_t)qi * p.H + h) * D + c) = acc;
}

template <int D>
cudaError_t launch_items_d(const AttnParams& p, int item_begin, int item_count, cudaStream_t stream, bool pdl) {
    using L = Smem<D>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    return launch_kernel(attn_kernel<D>, dim3((unsigned)item_count, (unsigned)p.Q), dim3(kThreads), L::kAlloc, stream,
                         pdl, p, item_begin);
}

}  // namespace

size_t attn_ws_bytes(int Q, int items, int d) {
    if (items <= 1) return 0;
    const size_t o = (size_t)Q * items * kHeadsPad * d * 4;
    const size_t l = (size_t)Q * items * kHeadsPad * 4;
    return ((o + 255) & ~(size_t)255) + ((l + 255) & ~(size_t)255);
}

void attn_ws_carve(AttnParams& p, void* ws) {
    if (p.n_items > 1) {
        const size_t o = (size_t)p.Q * p.n_items * kHeadsPad * p.d * 4;
        p.part_o = static_cast<float*>(ws);
        p.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + ((o + 255) & ~(size_t)255));
    }
}

cudaError_t launch_attention_items(const AttnParams& p, int item_begin, int item_count, cudaStream_t stream,
                                   bool pdl) {
    if (item_count <= 0) return cudaSuccess;
    if (p.d == 512) return launch_items_d<512>(p, item_begin, item_count, stream, pdl);
    if (p.d == 128) return launch_items_d<128>(p, item_begin, item_count, stream, pdl);
    return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const AttnParams& p, cudaStream_t stream, bool pdl) {
    if (p.n_items <= 1) return cudaSuccess;
    const dim3 grid((unsigned)p.H, (unsigned)p.Q);
    if (p.d == 512) return launch_kernel(combine_kernel<512>, grid, dim3(128), 0, stream, pdl, p);
    if (p.d == 128) return launch_kernel(combine_kernel<128>, grid, dim3(32), 0, stream, pdl, p);
    return cudaErrorInvalidValue;
}

}  // namespace csa

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
//     P   = exp2(S*scale*log2e - m)  (online softmax; four lanes share two rows)
//     O  += P . V             (64 heads x d, contraction over 64 keys)    tcgen05, M=64 N=256/128
// and writes either the final normalized output (single item) or a partial (O / l, lse) that
// combine_kernel merges by log-sum-exp.  The CSA/HCA merge of the method is exactly that merge.
//
// Layout: with M = 64 a head row lives in one 16-lane half of its warp's TMEM sub-partition.
// Lanes 0-15 hold Q (the A operand of Q.K^T, two bf16 per column) and two S buffers; lanes 16-31
// hold the fp32 O accumulator over all d columns.  Each key tile [64 x d] lives in shared memory
// as 128-byte-swizzled K-major blocks of 64 rows x 64 bf16 and doubles as the MN-major B operand
// of the P.V product, so every key is loaded once.  P is double-buffered in shared memory.
//
// Warp roles: warps 0-3 softmax + epilogue (O from TMEM straight to global memory), warps 4-7
// loaders (cp.async for gathered rows with manual swizzle and zero-fill of masked slots; TMA for
// full tiles of consecutive cache rows), warp 8 TMEM allocator + Q.K^T issuer, warp 9 P.V issuer.
// Three key stages; every wait is bounded (kWaitLimitNs) and winds the CTA down on timeout.
//
// Persistent CTAs (direct outputs of more queries than SMs, the PERSIST instantiation): one CTA per
// SM takes every G-th query of the launch; the key-stage ring, the S and P buffers and all barrier
// phases run on from one query to the next (a running tile count), the CTA's queries are set up
// once in shared memory, and the loader warps store each later query's Q (they own the same TMEM
// lane quarters as the softmax warps) once the previous query's last Q.K^T is done (q_empty).
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tma.h"

namespace csa {

namespace {

constexpr int kHeadsPad = 64;  // M of every MMA (heads beyond H are zero rows)
constexpr int kMaxCluster = 8; // CTAs of a decode cluster that merge their results
constexpr int kTileKeys = 64;
constexpr int kStages = 3;     // key tiles in flight
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
// TMEM map.  With M = 64 a head row lives in one half (16 lanes) of its warp's 32-lane
// sub-partition; the Q.K^T operands that share lanes 0-15 and the O accumulator in lanes 16-31
// together fill all 512 columns:
//   lanes 0-15:  Q (the A operand of Q.K^T, 2 bf16 per column) in columns [0, D/2),
//                S buffers b = 0, 1 in columns kColS + 64 b
//   lanes 16-31: O, dims [0, D) in columns [0, D)
constexpr uint32_t kColS = 256;
constexpr uint32_t kLaneO = 16;

// Per-CTA constants of the key list [CSA slots | raw window | HCA entries] of one query.
struct KeyList {
    const int32_t* idx;      // this query's k slots
    int64_t n_causal;        // floor(L / m)
    int64_t n_hca;           // floor(L / m') (0 without HCA)
    int64_t win_row0;        // raw row of the first window token
    int64_t nw;              // window tokens present
    int64_t csa_row0, hca_row0;
};

// One query of a CTA: its key list, the slice [s0, s1) of it the CTA attends and its key tiles.
struct QWork {
    KeyList kl;
    int64_t s0, s1;
    int T;
    int qi;
};
constexpr int kMaxQ = 64;  // queries of one persistent CTA (the launcher sizes the grid for it)

// NQ: queries a persistent CTA holds in shared memory (kMaxQ; 0 for the single-query kernel, which
// keeps its one query in registers)
template <int D, int NQ>
struct Smem {
    static constexpr int NKB = D / 64;                 // 64-wide blocks along d
    static constexpr int kBlock = 64 * 128;            // one block: 64 rows x 128 bytes
    static constexpr int kStage = NKB * kBlock;        // one key tile
    static constexpr int kK = 0;                       // kStages key tiles
    static constexpr int kP0 = kK + kStages * kStage;  // P, double-buffered
    static constexpr int kP1 = kP0 + kBlock;
    static constexpr int kBar = kP1 + kBlock;          // mbarriers
    static constexpr int kMisc = kBar + 32 * 8;        // tmem base, abort flag, masks
    static constexpr int kRowPtr = kMisc + 64;         // per loader warp: 16 row pointers
    static constexpr int kRowScl = kRowPtr + 4 * 16 * 8;  // and their FP4 scale rows (null: a bf16 row)
    static constexpr int kQTab = kRowScl + 4 * 16 * 8;  // the CTA's queries (QWork)
    static constexpr int kTotal = kQTab + NQ * (int)sizeof(QWork);
    static constexpr int kAlloc = kTotal + 1024;       // slack for 1024-byte alignment
    // cluster merge: the CTA's [64 x D] fp32 result in the freed key stages, rows padded by 16 bytes
    // so that the eight rows a warp's quads store hit different banks
    static constexpr int kOStride = D + 4;
    static_assert(64 * kOStride * 4 <= kStages * kStage, "the result fits in the key stages");
    static_assert(kBlock >= (64 + 16 * 64 + 64) * 4, "merge weights fit in the P buffers");
};

struct Bars {
    uint64_t full[kStages];   // loaders -> MMA / softmax: key stage holds tile t
    uint64_t empty[kStages];  // MMA commit after P.V of the tile in the stage
    uint64_t s_full[2];       // MMA commit after Q.K^T of tile t into S buffer t&1
    uint64_t s_free[2];       // softmax finished reading S buffer t&1
    uint64_t p_full[2];       // softmax wrote P buffer t&1 (and rescaled O if needed)
    uint64_t o_done[2];       // MMA commit after the P.V that read P buffer t&1
    uint64_t q_full;          // softmax warps stored Q in TMEM (once per query)
    uint64_t q_empty;         // MMA commit after the last Q.K^T of a query: the Q region is free
    uint64_t fin;             // both MMA issuers committed before teardown
};

// Tensor maps of the HCA cache and of the raw latents (boxes of 64 rows x 64 bf16, 128-byte swizzle).
struct AttnMaps {
    CUtensorMap hca;
    CUtensorMap x;
};


// Row pointer of slot `s` (nullptr = masked slot).
// The source of key s: a bf16 row (returned, *scl = nullptr) or, for an entry of a cache held in FP4,
// its code row (returned) with its scale row in *scl; nullptr for an empty or invalid slot.
__device__ __forceinline__ const void* key_src(const AttnParams& p, int D, const KeyList& kl, int64_t s,
                                               const uint8_t** scl, bool have_j = false, int32_t jpre = 0) {
    *scl = nullptr;
    if (s < p.k_slots) {
        const int32_t j = have_j ? jpre : kl.idx[s];  // the slot's index, unless the caller read it already
        if (j < 0) return nullptr;
        if ((int64_t)j >= kl.n_causal) {
            report(p.status, CSA_ERR_INDEX);
            return nullptr;
        }
        const int64_t r = kl.csa_row0 + j;
        if (p.entries_q) {
            *scl = p.entries_s + r * (D / 32);
            return p.entries_q + r * (D / 2);
        }
        return p.entries + r * D;
    }
    s -= p.k_slots;
    if (s < p.W) return s < kl.nw ? p.raw + (kl.win_row0 + s) * D : nullptr;
    s -= p.W;
    if (s >= kl.n_hca) return nullptr;
    const int64_t r = kl.hca_row0 + s;
    if (p.hca_q) {
        *scl = p.hca_s + r * (D / 32);
        return p.hca_q + r * (D / 2);
    }
    return p.hca + r * D;
}

// FP4: the instantiation for FP4 entry caches (its loaders dequantize FP4 rows); the other holds no
// FP4 code at all, which keeps the bf16 kernel's hot loops compact.  PERSIST: the instantiation for
// persistent CTAs over many queries (direct outputs); the other serves one (query, item) per CTA.
template <int D, bool FP4, bool PERSIST>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnMaps maps, AttnParams p,
                                                           int p_item_base) {
    using L = Smem<D, PERSIST ? kMaxQ : 0>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Bars* bars = reinterpret_cast<Bars*>(sm + L::kBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::kMisc);  // [0] tmem base, [1] abort, [2..7] masks
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    uint16_t* mask16 = reinterpret_cast<uint16_t*>(misc + 2);     // [stage][4 warps]
    const uint32_t sbase = smem_u32(sm);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int qi0 = blockIdx.y, item = blockIdx.x + p_item_base;
    if (p.hca_first) {
        const int n_hca = p.n_items - p.items_front;
        const int lin = blockIdx.x;
        if (lin < p.Q * n_hca) {
            qi0 = lin / n_hca;
            item = p.items_front + lin % n_hca;
        } else {
            qi0 = (lin - p.Q * n_hca) / p.items_front;
            item = (lin - p.Q * n_hca) % p.items_front;
        }
    }
    const int n_items = p.n_items;
    const bool direct = n_items == 1;
    // A direct launch with q_step > 0 is persistent: the CTA takes queries qi0, qi0 + q_step, ... and
    // its pipeline (key stages, S and P buffers, barrier phases) runs on from one query to the next,
    // so that the next query's key loads and Q.K^T products overlap this query's epilogue.
    const int q_step = (PERSIST && direct) ? p.q_step : 0;
    // (the launcher sizes the grid so that no CTA holds more than kMaxQ queries)
    const int n_q = q_step > 0 ? (qi0 < p.Q ? min((p.Q - 1 - qi0) / q_step + 1, kMaxQ) : 0) : 1;
    const bool clustered = !direct && p.cluster > 1;
    const bool dep_wait = !(p.hca_nowait && !direct && item >= p.items_front);
    // front items with a ready word: the loaders poll it, nobody waits for the select grid up front
    const bool ready_wait = dep_wait && p.ready != nullptr && !direct;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->full[i], 128);
            mbar_init(&bars->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->s_free[i], 128);
            mbar_init(&bars->p_full[i], 128);
            mbar_init(&bars->o_done[i], 1);
        }
        mbar_init(&bars->q_full, 128);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->fin, 2);
        misc[1] = 0;
        fence_mbar_init();
    }
    // The query table and sequence lengths: in the decode chain with an indexer they come from the
    // append two launches back, complete once this grid runs (every kernel of the chain waits before
    // it lets the next start); otherwise the previous launch may still be writing them.
    if (!p.queries_early) grid_dep_wait();
    // The key list of query qi and the slice [s0, s1) of it that this CTA attends; returns its number
    // of key tiles.
    const int64_t front = (int64_t)p.k_slots + p.W;
    auto work = [&](int qi, KeyList& kl, int64_t& s0, int64_t& s1) -> int {
        const csa_query qr = p.queries[qi];
        const bool seq_ok = qr.seq >= 0 && qr.reserved == 0;
        const csa_seq sq = seq_ok ? p.seqs[qr.seq] : csa_seq{0, 0, 0, 0};
        const bool qvalid = seq_ok && qr.len >= 1 && qr.len <= sq.len;
        kl.idx = p.idx ? p.idx + (int64_t)qi * p.k_slots : nullptr;
        kl.n_causal = qr.len / p.m;
        kl.n_hca = (p.use_hca && qvalid) ? qr.len / p.m_hca : 0;
        kl.nw = qr.len < p.W ? qr.len : p.W;
        kl.win_row0 = sq.tok_off + qr.len - kl.nw;
        kl.csa_row0 = sq.csa_off;
        kl.hca_row0 = sq.hca_off;
        const int64_t n_keys = front + kl.n_hca;
        if (direct) {
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
            if (item == 0 && (PERSIST || threadIdx.x == 0)) report(p.status, CSA_ERR_INDEX);
            s1 = s0;
        }
        // once any CTA has given up on a wait, later queries get no work (bounded total time on a fault)
        if (p.status && *reinterpret_cast<volatile int*>(p.status) == CSA_ERR_TIMEOUT) s1 = s0;
        return s1 > s0 ? (int)((s1 - s0 + kTileKeys - 1) / kTileKeys) : 0;
    };
    // The queries of a persistent CTA, evaluated once (one thread per query) into shared memory, so
    // that all roles cut the same key lists; a single query is evaluated by every thread (registers).
    QWork* qtab = reinterpret_cast<QWork*>(sm + L::kQTab);
    QWork w0{};
    if constexpr (PERSIST) {
        for (int jj = threadIdx.x; jj < n_q; jj += kThreads) {
            QWork w;
            w.qi = qi0 + jj * q_step;
            w.T = work(w.qi, w.kl, w.s0, w.s1);
            qtab[jj] = w;
        }
    } else {
        w0.qi = qi0;
        w0.T = work(qi0, w0.kl, w0.s0, w0.s1);
    }
    auto query = [&](int j) -> const QWork& {
        if constexpr (PERSIST) return qtab[j];
        return w0;
    };
    if (warp == 8 && n_q > 0) {
        tmem_alloc(misc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int T0 = n_q > 0 ? query(0).T : 0;
    // tensor-core work: any query of a persistent CTA may have key tiles
    const bool use_tc = q_step > 0 ? n_q > 0 : T0 > 0;

    // Q of query qi into TMEM, by the four warps of one role (warp w writes lane quarter w % 4), in
    // the A layout of Q.K^T: head row 16w + r in lane r of sub-partition w, dims 2c and 2c + 1 in
    // column c.  Written with the 16x256b shape, so every lane takes part: lane i writes rows i/4 and
    // i/4 + 8 at columns 8k + 2(i%4) and 8k + 2(i%4) + 1, i.e. 8 bytes of each of those rows per 8
    // columns.  The softmax warps store the first query's Q (an input, so before the wait on the
    // previous launch); the loaders store the j-th one (j > 0) of a persistent CTA once the products
    // of query j - 1 are done with the region (q_empty), its loads issued before that wait.
    auto load_q = [&](int qi, int j) -> bool {
        const int qw = warp & 3;
        const uint32_t q_lanes = (uint32_t)(qw * 32) << 16;
        const int qa = lane >> 2, qc = (lane & 3) * 2;
        const int h0 = qw * 16 + qa, h1 = h0 + 8;
        const uint2* q0 = reinterpret_cast<const uint2*>(p.q + ((int64_t)qi * p.H + (h0 < p.H ? h0 : 0)) * D);
        const uint2* q1 = reinterpret_cast<const uint2*>(p.q + ((int64_t)qi * p.H + (h1 < p.H ? h1 : 0)) * D);
        // optional RMS normalization of each head's query (gain p.q_norm): the four lanes of a quad
        // hold a quarter of the row each; a first pass sums the squares, the second scales
        float inv0 = 1.f, inv1 = 1.f;
        if (p.q_norm) {
            float ss0 = 0.f, ss1 = 0.f;
#pragma unroll 4
            for (int cb = 0; cb < D / 2; cb += 64) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int col = cb + 8 * k + qc;
                    float f[4];
                    const uint2 v0 = h0 < p.H ? q0[col / 2] : make_uint2(0, 0);
                    const uint2 v1 = h1 < p.H ? q1[col / 2] : make_uint2(0, 0);
                    f[0] = bf16lo(v0.x); f[1] = bf16hi(v0.x); f[2] = bf16lo(v0.y); f[3] = bf16hi(v0.y);
                    ss0 = fmaf(f[0], f[0], fmaf(f[1], f[1], fmaf(f[2], f[2], fmaf(f[3], f[3], ss0))));
                    f[0] = bf16lo(v1.x); f[1] = bf16hi(v1.x); f[2] = bf16lo(v1.y); f[3] = bf16hi(v1.y);
                    ss1 = fmaf(f[0], f[0], fmaf(f[1], f[1], fmaf(f[2], f[2], fmaf(f[3], f[3], ss1))));
                }
            }
            ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
            ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
            ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
            ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
            inv0 = rsqrtf(ss0 / D + p.norm_eps);
            inv1 = rsqrtf(ss1 / D + p.norm_eps);
        }
        const bool ok0 = h0 < p.H, ok1 = h1 < p.H;
        // dims 2col .. 2col + 3 of a row, normalized and rounded back to bf16 (gain p.q_norm)
        auto qnorm = [&](uint32_t& x, uint32_t& y, float inv, int col) {
            const float4 gn = *reinterpret_cast<const float4*>(p.q_norm + 2 * col);
            x = pack_bf16x2(bf16lo(x) * inv * gn.x, bf16hi(x) * inv * gn.y);
            y = pack_bf16x2(bf16lo(y) * inv * gn.z, bf16hi(y) * inv * gn.w);
        };
#pragma unroll 1
        for (int cb = 0; cb < D / 2; cb += 128) {
            uint32_t r[2][32];
            // every load of the pass first, unconditionally (a column past the row reads column
            // qc), so they are all in flight together; then the optional normalization and the
            // zeros of heads past H by selects on the loaded registers
#pragma unroll
            for (int g = 0; g < 2; ++g) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const bool in = cb + g * 64 < D / 2;
                    const int col = in ? cb + g * 64 + 8 * k + qc : qc;  // a column holds 2 dims
                    const uint2 v0 = q0[col / 2], v1 = q1[col / 2];
                    r[g][4 * k] = v0.x; r[g][4 * k + 1] = v0.y; r[g][4 * k + 2] = v1.x; r[g][4 * k + 3] = v1.y;
                }
            }
#pragma unroll
            for (int g = 0; g < 2; ++g) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const bool in = cb + g * 64 < D / 2;
                    const int col = in ? cb + g * 64 + 8 * k + qc : qc;
                    if (p.q_norm) {
                        qnorm(r[g][4 * k], r[g][4 * k + 1], inv0, col);
                        qnorm(r[g][4 * k + 2], r[g][4 * k + 3], inv1, col);
                    }
                    const bool u0 = in && ok0, u1 = in && ok1;
                    r[g][4 * k] = u0 ? r[g][4 * k] : 0u;
                    r[g][4 * k + 1] = u0 ? r[g][4 * k + 1] : 0u;
                    r[g][4 * k + 2] = u1 ? r[g][4 * k + 2] : 0u;
                    r[g][4 * k + 3] = u1 ? r[g][4 * k + 3] : 0u;
                }
            }
            if (cb == 0 && j > 0) {
                const bool w = mbar_wait(&bars->q_empty, (uint32_t)(j - 1) & 1u, p.status, abort_flag, p.wait_ns);
                if (!__all_sync(0xffffffffu, w)) return false;  // (the stores below are warp-collective)
                tc_fence_after();
            }
#pragma unroll
            for (int g = 0; g < 2; ++g)
                if (cb + g * 64 < D / 2) tmem_st_16x256_x8(tmem + q_lanes + (uint32_t)(cb + g * 64), r[g]);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->q_full);
        return true;
    };

    if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ loaders
        const int lw = warp - 4;
        const uint64_t* rowptr = reinterpret_cast<const uint64_t*>(sm + L::kRowPtr) + lw * 16;
        uint64_t* rowptr_w = reinterpret_cast<uint64_t*>(sm + L::kRowPtr) + lw * 16;
        const uint64_t* rowscl = reinterpret_cast<const uint64_t*>(sm + L::kRowScl) + lw * 16;
        uint64_t* rowscl_w = reinterpret_cast<uint64_t*>(sm + L::kRowScl) + lw * 16;
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        // Lane l copies 16-byte chunks l, l+32, ... of each 64-chunk (1 KiB) row: chunk c lands in
        // block c/8 at swizzled position (c%8) ^ (row%8), and c%8 = l%8 for every chunk of a lane.
        constexpr int CPL = CPR / 32 > 0 ? CPR / 32 : 1;  // chunks per lane per row (2 at D = 512)
        const uint32_t lane_blk = (uint32_t)(lane >> 3) * L::kBlock;  // block of chunk `lane`
        const uint32_t lane_c7 = (uint32_t)(lane & 7);
        // the selected indices come from the previous kernel: its ready word for this query, or the
        // end of its grid
        bool go = true;
        if (ready_wait) {
            if (lane == 0) go = count_wait(p.ready + qi0, 1u, p.status, abort_flag, p.wait_ns);
            __syncwarp();  // orders the other lanes' reads after lane 0's acquire
            go = __shfl_sync(0xffffffffu, go ? 1 : 0, 0) != 0;
        } else if (dep_wait) {
            grid_dep_wait();
        }
        if (lw == 0 && lane == 0) {
            if (p.tma_hca) tma_prefetch_map(&maps.hca);
            if (p.tma_x) tma_prefetch_map(&maps.x);
        }
        // per stage, the full-barrier parity of the last tile this thread loaded by TMA (bit 2 set:
        // one is pending), so that a CTA that gives up waits for its own copies before it exits
        uint32_t tma_pend = 0;
        uint32_t g = 0;  // key tiles of the CTA's earlier queries (the stage ring runs on)
        for (int j = 0; go && j < n_q; ++j) {
            const KeyList kl = query(j).kl;
            const int64_t s0 = query(j).s0, s1 = query(j).s1;
            const int T = query(j).T;
            // the selected index of this lane's row in tile t, read ahead: the first two tiles' together
            // (one memory latency, not one per tile), and in a persistent CTA, whose queries span many
            // tiles of slots, tile t + 2's while tile t is loaded, so that no tile waits on its indices
            // (a single-query CTA reads later tiles' indices as it loads them); an address past the
            // slots reads the last slot, unused
            const bool pre = kl.idx && lane < 16;
            auto read_j = [&](int t) -> int32_t {
                const int64_t tb = s0 + (int64_t)t * kTileKeys;
                if (!PERSIST && t >= 2) return -1;
                if (!pre || t >= T || tb >= p.k_slots) return -1;
                const int64_t sa = tb + lw * 16 + lane;
                return kl.idx[sa < p.k_slots ? sa : p.k_slots - 1];
            };
            int32_t j_next = read_j(0), j_after = read_j(1);
            for (int t = 0; t < T; ++t) {
                const int32_t j_t = j_next;
                j_next = j_after;
                j_after = read_j(t + 2);
                // a persistent CTA's next query: its Q goes into TMEM after the query's first tile is
                // issued (the products of the previous query still read the region until then)
                if (PERSIST && j > 0 && t == 1 && !load_q(query(j).qi, j)) {
                    go = false;
                    break;
                }
                const uint32_t gt = g + (uint32_t)t;
                const int st = (int)(gt % kStages);
                if (gt >= kStages &&
                    !mbar_wait(&bars->empty[st], ((gt / kStages) - 1) & 1, p.status, abort_flag, p.wait_ns)) {
                    go = false;
                    break;
                }
                const int64_t tb = s0 + (int64_t)t * kTileKeys;
                // A full tile of consecutive cache rows (HCA entries, or raw window tokens) goes by TMA:
                // one thread issues the boxes, the tile's bytes complete the full barrier, and the
                // loaders move on without waiting for the data.
                const CUtensorMap* map = nullptr;
                int64_t row = 0;
                if (tb + kTileKeys <= s1) {
                    if (p.tma_hca && tb >= front && tb - front + kTileKeys <= kl.n_hca) {
                        map = &maps.hca;
                        row = kl.hca_row0 + (tb - front);
                    } else if (p.tma_x && tb >= p.k_slots && tb - p.k_slots + kTileKeys <= kl.nw) {
                        map = &maps.x;
                        row = kl.win_row0 + (tb - p.k_slots);
                    }
                    if (row < 0 || row > 0x7FFFFFFF - kTileKeys) map = nullptr;
                }
                // fault injection (tests of the bounded waits): the first loader warp skips its arrival
                // on the first tile, which therefore never becomes full
                const bool skip = p.debug_fault == 1 && gt == 0 && lw == 0;
                if (map) {
                    if (lw == 0 && lane == 0) {
                        for (int w4 = 0; w4 < 4; ++w4) mask16[st * 4 + w4] = 0xFFFFu;
                        mbar_arrive_expect_tx(&bars->full[st], (uint32_t)(kTileKeys * D * 2));
                        const uint32_t kdst = sbase + L::kK + (uint32_t)st * L::kStage;
#pragma unroll
                        for (int kb = 0; kb < L::NKB; ++kb)
                            tma_load_2d(kdst + (uint32_t)kb * L::kBlock, map, kb * 64, (int)row, &bars->full[st]);
                        tma_pend = (tma_pend & ~(7u << (3 * st))) | ((4u | ((gt / kStages) & 1u)) << (3 * st));
                    } else if (!skip) {
                        mbar_arrive(&bars->full[st]);
                    }
                    continue;
                }
                bool valid = false, fp4 = false;
                if (lane < 16) {
                    const int64_t s = tb + lw * 16 + lane;
                    const uint8_t* scl = nullptr;
                    const void* r = s < s1 ? key_src(p, D, kl, s, &scl, pre && (PERSIST || t < 2), j_t) : nullptr;
                    rowptr_w[lane] = reinterpret_cast<uint64_t>(r);
                    rowscl_w[lane] = reinterpret_cast<uint64_t>(scl);
                    valid = r != nullptr;
                    fp4 = FP4 && scl != nullptr;
                }
                const uint32_t vm = __ballot_sync(0xffffffffu, valid) & 0xFFFFu;
                const bool tile_fp4 = __ballot_sync(0xffffffffu, fp4) != 0u;
                __syncwarp();
                const uint32_t kbase = sbase + L::kK + (uint32_t)st * L::kStage + lane_blk;
                // a bf16 row (or an empty one: zeros) by cp.async, this lane's 16-byte chunks
                auto copy_row = [&](int r) {
                    const uint16_t* row = reinterpret_cast<const uint16_t*>(rowptr[r]);
                    const int key = lw * 16 + r;
                    const uint32_t dst = kbase + (uint32_t)key * 128u + ((lane_c7 ^ (key & 7)) << 4);
                    const uint32_t nb = row ? 16u : 0u;
                    const uint16_t* src = row ? row : p.q;
                    if (CPR >= 32) {
#pragma unroll
                        for (int u = 0; u < CPL; ++u)
                            cp_async16(dst + u * 4 * L::kBlock, src + (lane + 32 * u) * 8, nb);
                    } else if (lane < CPR) {
                        cp_async16(dst, src + lane * 8, nb);
                    }
                };
                if (!FP4 || !tile_fp4) {
#pragma unroll 4
                    for (int r = 0; r < 16; ++r) copy_row(r);
                    // the copies complete the tile's barrier phase themselves: no wait here, so the next
                    // tile's loads go out while these are still in flight
                    if (!skip) cp_async_mbar_arrive(&bars->full[st]);
                } else {
                    // FP4 entries: chunk c of a row (channels 8c .. 8c+7) is the 4 code bytes at 4c and the
                    // scale byte c/4; dequantized in registers and stored into the tile's swizzled slot.
                    // The loads of all 16 rows are issued first, unconditionally (a row that is not FP4
                    // loads from the query instead and goes by cp.async), so the tile costs one memory
                    // latency; then the rows are converted.
                    constexpr int kFp4Rows = 16;
#pragma unroll 1
                    for (int r0 = 0; r0 < 16; r0 += kFp4Rows) {
                        uint32_t cw[kFp4Rows][CPL], sb[kFp4Rows][CPL];
#pragma unroll
                        for (int i = 0; i < kFp4Rows; ++i) {
                            const uint8_t* sc = reinterpret_cast<const uint8_t*>(rowscl[r0 + i]);
                            const uint8_t* cr = sc ? reinterpret_cast<const uint8_t*>(rowptr[r0 + i])
                                                   : reinterpret_cast<const uint8_t*>(p.q);
                            const uint8_t* sr = sc ? sc : reinterpret_cast<const uint8_t*>(p.q);
#pragma unroll
                            for (int u = 0; u < CPL; ++u) {
                                const int c = (lane + 32 * u) < CPR ? lane + 32 * u : 0;
                                cw[i][u] = __ldg(reinterpret_cast<const unsigned int*>(cr + 4 * c));
                                sb[i][u] = __ldg(sr + (c >> 2));
                            }
                        }
#pragma unroll
                        for (int i = 0; i < kFp4Rows; ++i) {
                            const int r = r0 + i;
                            if (rowscl[r] == 0) {
                                copy_row(r);
                                continue;
                            }
                            const int key = lw * 16 + r;
                            const uint32_t dst = kbase + (uint32_t)key * 128u + ((lane_c7 ^ (key & 7)) << 4);
#pragma unroll
                            for (int u = 0; u < CPL; ++u)
                                if (lane + 32 * u < CPR)
                                    st_shared_v4(dst + u * 4 * L::kBlock, mx4_to_bf16x8(cw[i][u], sb[i][u]));
                        }
                    }
                    cp_async_wait_all();
                    fence_proxy_async_smem();
                }
                if (lane == 0) mask16[st * 4 + lw] = (uint16_t)vm;
                __syncwarp();
                if (!skip) mbar_arrive(&bars->full[st]);
            }
            if (PERSIST && go && j > 0 && T <= 1 && !load_q(query(j).qi, j)) go = false;
            g += (uint32_t)T;
        }
        cp_async_wait_all();
        if (*abort_flag && tma_pend) {
            // the CTA gave up: its TMA copies may still be landing in shared memory; wait (bounded)
            // for the tiles whose barrier phase has not completed before the CTA exits
            for (int st = 0; st < kStages; ++st) {
                const uint32_t e = (tma_pend >> (3 * st)) & 7u;
                if (e & 4u) mbar_wait(&bars->full[st], e & 1u, nullptr, nullptr, p.wait_ns);
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------------ MMA issuers
        // warp 8 issues Q.K^T of every tile (A = Q from TMEM), warp 9 issues P.V (A = P, B = the key
        // tile read MN-major as V): the two products of neighbouring tiles reach the tensor pipe
        // independently, so a P.V never waits behind the issue of the next Q.K^T.  Each warp runs
        // its loop with all lanes (warp-uniform waits and operands; one elected lane issues).
        if (dep_wait && !ready_wait) grid_dep_wait();
        if (use_tc) {
            // g: key tiles of the CTA's earlier queries (stage, S and P buffer phases run on)
            uint32_t g = 0;
            bool ok = true;
            if (warp == 8) {
                constexpr uint32_t id1 = idesc_bf16(64, 64, false, false);
                for (int j = 0; ok && j < n_q; ++j) {
                    const int T = query(j).T;
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&bars->q_full, (uint32_t)j & 1u, p.status, abort_flag, p.wait_ns));
                    for (int t = 0; ok && t < T; ++t) {
                        const uint32_t gt = g + (uint32_t)t;
                        const int st = (int)(gt % kStages);
                        bool w = mbar_wait(&bars->full[st], (gt / kStages) & 1, p.status, abort_flag, p.wait_ns);
                        if (w && gt >= 2)
                            w = mbar_wait(&bars->s_free[gt & 1], ((gt >> 1) - 1) & 1, p.status, abort_flag, p.wait_ns);
                        if (!__all_sync(0xffffffffu, w)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        fence_proxy_async_smem();  // the tile's cp.async writes, observed through the barrier
                        const uint64_t kd = sdesc_kmajor(sbase + L::kK + (uint32_t)st * L::kStage);
                        const uint32_t tS = tmem + kColS + (gt & 1u) * 64u;
#pragma unroll
                        for (int kb = 0; kb < L::NKB; ++kb) {
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) {
                                // K elements [64 kb + 16 ks, +16): columns 32 kb + 8 ks of Q, bytes of the tile block
                                umma_bf16_ts(tS, tmem + (uint32_t)(kb * 32 + ks * 8),
                                             kd + (uint64_t)((kb * L::kBlock + ks * 32) >> 4), id1, (kb | ks) != 0);
                            }
                        }
                        umma_commit(&bars->s_full[gt & 1]);
                    }
                    // the query's products have read Q once this completes: the next Q may be stored
                    if (PERSIST) umma_commit(&bars->q_empty);
                    g += (uint32_t)T;
                }
            } else {
                constexpr int N2 = D >= 256 ? 256 : D;
                constexpr int HALVES = D >= 256 ? D / 256 : 1;
                constexpr uint32_t id2 = idesc_bf16(64, N2, false, true);
                for (int j = 0; ok && j < n_q; ++j) {
                    const int T = query(j).T;
                    for (int t = 0; t < T; ++t) {
                        const uint32_t gt = g + (uint32_t)t;
                        const bool w = mbar_wait(&bars->p_full[gt & 1], (gt >> 1) & 1, p.status, abort_flag, p.wait_ns);
                        if (!__all_sync(0xffffffffu, w)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const int st = (int)(gt % kStages);
                        const uint64_t vd = sdesc_mnmajor(sbase + L::kK + (uint32_t)st * L::kStage, L::kBlock);
                        const uint64_t pd = sdesc_kmajor(sbase + ((gt & 1u) ? L::kP1 : L::kP0));
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                            for (int half = 0; half < HALVES; ++half) {
                                // V rows ks*16 .. ks*16+15 of the key tile, dims [half*256, half*256 + N2);
                                // the query's first product overwrites O
                                const uint64_t b = vd + (uint64_t)((half * 4 * L::kBlock + ks * 16 * 128) >> 4);
                                const uint32_t tO = tmem + (kLaneO << 16) + (uint32_t)(half * 256);
                                umma_bf16(tO, pd + (uint64_t)((ks * 32) >> 4), b, id2, (t > 0 || ks > 0) ? 1u : 0u);
                            }
                        }
                        umma_commit(&bars->empty[st]);
                        umma_commit(&bars->o_done[gt & 1]);
                    }
                    g += (uint32_t)T;
                }
            }
            umma_commit(&bars->fin);
            mbar_wait(&bars->fin, 0, p.status, nullptr, p.wait_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax + epilogue
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t o_base = tmem + lane_base + (kLaneO << 16);
        bool ok = true;
        if (use_tc) ok = load_q(qi0, 0);
        if (dep_wait && !ready_wait) grid_dep_wait();
        grid_dep_launch();
        const int i = lane;
        // S and O are read with the 16x256b shape, so all 32 lanes work: lane i holds rows ra = i/4
        // and ra + 8 of the warp's 16, at columns 8k + cq and 8k + cq + 1 of every 64-column group;
        // the four lanes of a quad share a row and combine their partial max / sum by shuffles.
        const int ra = i >> 2, cq = (i & 3) * 2;
        const int hr[2] = {warp * 16 + ra, warp * 16 + ra + 8};
        uint32_t g = 0;  // key tiles of the CTA's earlier queries
        for (int j = 0; j < n_q; ++j) {
            const int qi = query(j).qi;
            const int T = query(j).T;
            float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
            for (int t = 0; ok && t < T; ++t) {
                const uint32_t gt = g + (uint32_t)t;
                const int sb = (int)(gt & 1u), st = (int)(gt % kStages);
                ok = mbar_wait(&bars->s_full[sb], (gt >> 1) & 1, p.status, abort_flag, p.wait_ns) &&
                     mbar_wait(&bars->full[st], (gt / kStages) & 1, p.status, abort_flag, p.wait_ns);
                if (!ok) break;
                tc_fence_after();
                float s[2][16];  // [row ra / ra+8][2k + e] = column 8k + cq + e
                {
                    uint32_t r[32];
                    tmem_ld_16x256_x8(tmem + lane_base + kColS + (uint32_t)sb * 64u, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        s[0][2 * k] = __uint_as_float(r[4 * k]);
                        s[0][2 * k + 1] = __uint_as_float(r[4 * k + 1]);
                        s[1][2 * k] = __uint_as_float(r[4 * k + 2]);
                        s[1][2 * k + 1] = __uint_as_float(r[4 * k + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->s_free[sb]);
                const uint64_t vmask = (uint64_t)mask16[st * 4 + 0] | ((uint64_t)mask16[st * 4 + 1] << 16) |
                                       ((uint64_t)mask16[st * 4 + 2] << 32) | ((uint64_t)mask16[st * 4 + 3] << 48);
                const float sc = p.scale_log2;
                float mx[2] = {-INFINITY, -INFINITY};
                const uint64_t lm = vmask >> cq;  // bit 8k + e: column 8k + cq + e valid
#pragma unroll
                for (int k = 0; k < 8; ++k) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool v = (lm >> (8 * k + e)) & 1ull;
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            s[rr][2 * k + e] = v ? s[rr][2 * k + e] * sc : -INFINITY;
                            mx[rr] = fmaxf(mx[rr], s[rr][2 * k + e]);
                        }
                    }
                }
                float alpha[2] = {1.f, 1.f};
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
                    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
                    // lazy rescaling: move the reference max only when it grows by more than 2^8
                    if (mx[rr] > m_run[rr] + 8.f) {
                        alpha[rr] = (m_run[rr] == -INFINITY) ? 0.f : exp2f(m_run[rr] - mx[rr]);
                        m_run[rr] = mx[rr];
                        l_run[rr] *= alpha[rr];
                    }
                }
                // O must hold every earlier P.V before it is rescaled (rare); O lives in lanes 16-31,
                // in the same row / column layout as S
                const bool any = __any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f);
                if (t > 0 && any) {
                    ok = mbar_wait(&bars->o_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, p.status, abort_flag, p.wait_ns);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D; c += 64) {
                        uint32_t r[32];
                        tmem_ld_16x256_x8(o_base + (uint32_t)c, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            r[4 * k] = __float_as_uint(__uint_as_float(r[4 * k]) * alpha[0]);
                            r[4 * k + 1] = __float_as_uint(__uint_as_float(r[4 * k + 1]) * alpha[0]);
                            r[4 * k + 2] = __float_as_uint(__uint_as_float(r[4 * k + 2]) * alpha[1]);
                            r[4 * k + 3] = __float_as_uint(__uint_as_float(r[4 * k + 3]) * alpha[1]);
                        }
                        tmem_st_16x256_x8(o_base + (uint32_t)c, r);
                    }
                    tmem_st_wait();
                }
                // P buffer t&1 is free once the P.V of tile t-2 finished
                if (gt >= 2) {
                    ok = mbar_wait(&bars->o_done[sb], ((gt >> 1) - 1) & 1, p.status, abort_flag, p.wait_ns);
                    if (!ok) break;
                }
                {
                    // masked slots hold -inf: 2^(-inf - m) = 0; while a row has seen no key, m_use = 0
                    const uint32_t prow = sbase + (sb ? L::kP1 : L::kP0) + (uint32_t)(i & 3) * 4u;
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const float m_use = m_run[rr] == -INFINITY ? 0.f : m_run[rr];
                        float lsum = 0.f;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float p0 = fast_exp2(s[rr][2 * k] - m_use);
                            const float p1 = fast_exp2(s[rr][2 * k + 1] - m_use);
                            lsum += p0 + p1;
                            asm volatile("st.shared.b32 [%0], %1;" ::"r"(prow + sw128_offset(hr[rr], k)),
                                         "r"(pack_bf16x2(p0, p1))
                                         : "memory");
                        }
                        l_run[rr] += lsum;  // this lane's part of the row sum; the quad adds them up at the end
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bars->p_full[sb]);
            }
            const int Tq = T;
            const uint32_t gq = g;
            g += (uint32_t)T;
            // ---- epilogue: TMEM -> registers -> global memory
            if (ok && Tq > 0) {
                const uint32_t gl = gq + (uint32_t)Tq - 1u;
                ok = mbar_wait(&bars->o_done[gl & 1], (gl >> 1) & 1, p.status, abort_flag, p.wait_ns);
            }
            float inv[2], lse2[2];  // lse2: log-sum-exp in log2 units
            bool has[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
                l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
                has[rr] = ok && Tq > 0 && l_run[rr] > 0.f;
                inv[rr] = has[rr] ? 1.f / l_run[rr] : 0.f;
                lse2[rr] = has[rr] ? m_run[rr] + log2f(l_run[rr]) : -INFINITY;
                // a single item holds the query's whole softmax: its sink logit (one more term with a zero
                // value) joins here; with several items it joins in the merge
                const float z = (direct && p.sink && hr[rr] < p.H) ? p.sink[hr[rr]] * 1.4426950408889634f : -INFINITY;
                if (z > -INFINITY && (ok || Tq == 0)) {
                    const float m_eff = has[rr] ? fmaxf(m_run[rr], z) : z;
                    const float a = has[rr] ? exp2f(m_run[rr] - m_eff) : 0.f;
                    const float l_eff = fmaf(l_run[rr], a, exp2f(z - m_eff));
                    inv[rr] = a / l_eff;
                    lse2[rr] = m_eff + log2f(l_eff);
                }
            }
            const bool write_o = ok && Tq > 0;
            const int rows = p.H < kHeadsPad ? p.H : kHeadsPad;
            const bool to_smem = clustered;  // the cluster merges its CTAs' results in shared memory
            float* o_smem = reinterpret_cast<float*>(sm + L::kK);
            if (write_o) {
                // straight from the registers: per row, the four lanes of a quad write 32 consecutive
                // bytes (one full sector) per instruction
                float* dst[2];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
                    dst[rr] = to_smem ? o_smem + hr[rr] * L::kOStride
                              : direct ? p.out + ((int64_t)qi * p.H + hr[rr]) * D
                                       : p.part_o + (((int64_t)qi * n_items + item) * kHeadsPad + hr[rr]) * D;
                tc_fence_after();
                // two register buffers: the TMEM load of the next 64 columns is in flight while the
                // current ones are stored
                auto store64 = [&](const uint32_t (&r)[32], int c) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int col = c + 8 * k + cq;
                        if (hr[0] < rows)
                            *reinterpret_cast<float2*>(dst[0] + col) =
                                make_float2(__uint_as_float(r[4 * k]) * inv[0], __uint_as_float(r[4 * k + 1]) * inv[0]);
                        if (hr[1] < rows)
                            *reinterpret_cast<float2*>(dst[1] + col) = make_float2(__uint_as_float(r[4 * k + 2]) * inv[1],
                                                                                 __uint_as_float(r[4 * k + 3]) * inv[1]);
                    }
                };
                static_assert(D % 128 == 0, "column chunks come in pairs");
                uint32_t ra[32], rb[32];
                tmem_ld_16x256_x8(o_base, ra);
                tmem_ld_wait();
#pragma unroll 1
                for (int c = 0; c < D; c += 128) {
                    tmem_ld_16x256_x8(o_base + (uint32_t)(c + 64), rb);
                    store64(ra, c);
                    tmem_ld_wait();
                    if (c + 128 < D) tmem_ld_16x256_x8(o_base + (uint32_t)(c + 128), ra);
                    store64(rb, c + 64);
                    tmem_ld_wait();
                }
            } else if (direct) {
                const int tid = threadIdx.x;  // 0..127
                for (int e = tid; e < rows * (D / 4); e += 128) {
                    const int hh = e / (D / 4), c4 = e % (D / 4);
                    *reinterpret_cast<float4*>(p.out + ((int64_t)qi * p.H + hh) * D + c4 * 4) =
                        make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if ((i & 3) == 0) {
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int h = hr[rr];
                    if (h >= p.H) continue;
                    const float lse_v = lse2[rr] * 0.69314718055994531f;
                    if (direct) {
                        if (p.lse) p.lse[(int64_t)qi * p.H + h] = lse_v;
                    } else if (to_smem) {
                        reinterpret_cast<float*>(sm + L::kP0)[h] = lse_v;
                    } else {
                        p.part_lse[((int64_t)qi * n_items + item) * kHeadsPad + h] = lse_v;
                    }
                }
                if (to_smem && (i & 3) == 0)  // rows of heads past H: no contribution
                    for (int rr = 0; rr < 2; ++rr)
                        if (hr[rr] >= p.H) reinterpret_cast<float*>(sm + L::kP0)[hr[rr]] = -INFINITY;
            }
        }  // queries of the CTA
    }
    // the select grid is complete before this one is (the merge that waits for this grid relies on it)
    if (ready_wait) grid_dep_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 8 && n_q > 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (clustered) {
        // ---- the cluster's merge: CTA `rank` combines columns [rank * D/F, (rank + 1) * D/F) of the
        // F results (each normalized by its own sum, with its lse) into one partial of the query
        const int F = p.cluster;
        const uint32_t rank = cluster_ctarank();
        const float* o_smem = reinterpret_cast<const float*>(sm + L::kK);  // [64][kOStride] results
        float* lse_s = reinterpret_cast<float*>(sm + L::kP0);        // [64] this CTA's lse
        float* wts = lse_s + kHeadsPad;                               // [F][64] merge weights
        float* mlse = wts + F * kHeadsPad;                            // [64] merged lse
        // (the softmax warps wrote lse_s for all 64 rows: -inf for rows without a result, so an
        // empty or failed CTA contributes nothing and its unwritten rows are never read)
        cluster_barrier();
        if (threadIdx.x < kHeadsPad) {
            const int h = threadIdx.x;
            float l[kMaxCluster];
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) l[c] = c < F ? ld_cluster_f32(lse_s + h, (uint32_t)c) : -INFINITY;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) mx = fmaxf(mx, l[c]);
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) {
                l[c] = mx == -INFINITY ? 0.f : expf(l[c] - mx);
                sum += l[c];
            }
            for (int c = 0; c < F; ++c) wts[c * kHeadsPad + h] = sum > 0.f ? l[c] / sum : 0.f;
            mlse[h] = mx == -INFINITY ? -INFINITY : mx + logf(sum);
        }
        __syncthreads();
        const int cols = D / F, n4 = cols / 4;
        const int part = item / F;
        const int n_parts = n_items / F;
        // every load of an output's F contributions is issued before any of them is used (the
        // remote shared-memory latency is paid once per output, not once per contribution)
        for (int e = threadIdx.x; e < kHeadsPad * n4; e += kThreads) {
            const int h = e / n4, col = (int)rank * cols + 4 * (e % n4);
            float4 v[kMaxCluster];
            float w[kMaxCluster];
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) {
                w[c] = c < F ? wts[c * kHeadsPad + h] : 0.f;
                v[c] = w[c] > 0.f ? ld_cluster_f32x4(o_smem + h * L::kOStride + col, (uint32_t)c)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) {
                acc.x = fmaf(w[c], v[c].x, acc.x);
                acc.y = fmaf(w[c], v[c].y, acc.y);
                acc.z = fmaf(w[c], v[c].z, acc.z);
                acc.w = fmaf(w[c], v[c].w, acc.w);
            }
            if (h < p.H)
                *reinterpret_cast<float4*>(p.part_o + (((int64_t)qi0 * n_parts + part) * kHeadsPad + h) * D + col) =
                    acc;
        }
        if (rank == 0)
            for (int h = threadIdx.x; h < kHeadsPad; h += kThreads)
                p.part_lse[((int64_t)qi0 * n_parts + part) * kHeadsPad + h] = mlse[h];
        cluster_barrier();  // no CTA leaves while another still reads its shared memory
    }
    if (p.items_done && !direct) {
        __syncthreads();  // every partial store of the CTA precedes the count
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(p.items_done + qi0, 1u);
        }
    }
}

// out[q][h] = sum_items exp(lse_i - lse) * O_i,  lse = logsumexp_i lse_i  (items with lse = -inf
// contribute nothing and are not read).  One CTA per (head, query, 1/SPLIT of the dims); warp 0
// computes the weights, then every thread accumulates one float4 column of all contributing
// partials with batched loads.
template <int D, int SPLIT>
__global__ void combine_kernel(AttnParams p) {
    constexpr int kMaxBatch = 32;  // partial rows held in registers per pass
    const int h = blockIdx.x, qi = blockIdx.y;
    const int n_items = p.cluster > 1 ? p.n_items / p.cluster : p.n_items;  // partials per query
    const int lane = threadIdx.x & 31;
    __shared__ float s_lse[256];
    __shared__ float s_w[256];
    __shared__ float s_res[2];
    __shared__ int s_go;
    // the partials come from the attention grid: this query's item counter, or the end of the grid
    if (p.items_done) {
        if (threadIdx.x == 0) s_go = count_wait(p.items_done + qi, (uint32_t)p.n_items, p.status, nullptr, p.wait_ns);
        __syncthreads();  // orders every thread's reads after thread 0's acquire
        if (!s_go) {
            grid_dep_wait();
            return;
        }
    } else {
        grid_dep_wait();
    }
    // every thread owns one float4 column of the output row (D / 4 / SPLIT threads)
    const int c = (int)blockIdx.z * (D / SPLIT) + threadIdx.x * 4;
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
        // the head's sink logit, if any: one more softmax term whose value is zero
        const float z = p.sink ? p.sink[h] : -INFINITY;
        float mx = z;
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
        if (z > -INFINITY) sum += expf(z - mx);
        if (lane == 0) {
            s_res[0] = sum > 0.f ? 1.f / sum : 0.f;
            s_res[1] = mx == -INFINITY ? -INFINITY : mx + logf(sum);
        }
    }
    __syncthreads();
    const float inv = s_res[0];
    if (threadIdx.x == 0 && blockIdx.z == 0 && p.lse) p.lse[(int64_t)qi * p.H + h] = s_res[1];
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

// Multiprocessors of the current device (0 if unknown), cached per device.
int device_sms() {
    static std::atomic<int> counts[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int v = counts[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        counts[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

template <int D>
cudaError_t launch_items_d(const AttnParams& p, int item_begin, int item_count, cudaStream_t stream, bool pdl) {
    using L = Smem<D, 0>;
    using LP = Smem<D, kMaxQ>;
    static PerDeviceOnce attr;
    cudaError_t ea = attr.run([] {
        constexpr auto a = cudaFuncAttributeMaxDynamicSharedMemorySize;
        cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, false, false>, a, L::kAlloc);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_kernel<D, true, false>, a, L::kAlloc);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_kernel<D, false, true>, a, LP::kAlloc);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_kernel<D, true, true>, a, LP::kAlloc);
        return e;
    });
    if (ea != cudaSuccess) return ea;
    const bool fp4 = p.entries_q || p.hca_q;
    auto kernel = fp4 ? attn_kernel<D, true, false> : attn_kernel<D, false, false>;
    dim3 grid = p.hca_first ? dim3((unsigned)(p.n_items * p.Q)) : dim3((unsigned)item_count, (unsigned)p.Q);
    // tensor maps over the HCA cache and the raw latents; the kernel only issues boxes that lie
    // inside one sequence's valid rows, so the row extent is left open
    AttnMaps maps;
    AttnParams q = p;
    q.tma_hca = p.use_hca && p.hca && !p.hca_q &&
                tensor_map_2d_bf16(&maps.hca, p.hca, D, 0x7FFFFFFFull, (uint64_t)D * 2, 64, kTileKeys) == cudaSuccess;
    q.tma_x = p.raw && p.W >= kTileKeys &&
              tensor_map_2d_bf16(&maps.x, p.raw, D, 0x7FFFFFFFull, (uint64_t)D * 2, 64, kTileKeys) == cudaSuccess;
    if (!q.tma_hca) std::memset(&maps.hca, 0, sizeof(maps.hca));
    if (!q.tma_x) std::memset(&maps.x, 0, sizeof(maps.x));
    // direct outputs: persistent CTAs, one per SM (one fits, by its shared and tensor memory) or
    // more when a CTA would otherwise hold over kMaxQ queries, each taking every G-th query, so that
    // a query's epilogue overlaps the next one's first products
    q.q_step = 0;
    int smem = L::kAlloc;
    if (p.persist && p.n_items == 1 && !p.hca_first && p.cluster <= 1 && item_count == 1) {
        const int sms = device_sms();
        const int G = sms > (p.Q + kMaxQ - 1) / kMaxQ ? sms : (p.Q + kMaxQ - 1) / kMaxQ;
        if (sms > 0 && p.Q > G) {
            q.q_step = G;
            grid = dim3(1u, (unsigned)G);
            kernel = fp4 ? attn_kernel<D, true, true> : attn_kernel<D, false, true>;
            smem = LP::kAlloc;
        }
    }
    if (q.cluster > 1 && q.n_items > 1)
        return launch_kernel_cluster(kernel, grid, dim3(kThreads), smem, stream, pdl,
                                     dim3((unsigned)q.cluster, 1, 1), maps, q, item_begin);
    return launch_kernel(kernel, grid, dim3(kThreads), smem, stream, pdl, maps, q, item_begin);
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
    // 512 dims: two CTAs of 64 threads per (head, query), so the merge spreads over more SMs
    if (p.d == 512)
        return launch_kernel(combine_kernel<512, 2>, dim3((unsigned)p.H, (unsigned)p.Q, 2), dim3(64), 0, stream, pdl, p);
    if (p.d == 128)
        return launch_kernel(combine_kernel<128, 1>, dim3((unsigned)p.H, (unsigned)p.Q, 1), dim3(32), 0, stream, pdl, p);
    return cudaErrorInvalidValue;
}

}  // namespace csa

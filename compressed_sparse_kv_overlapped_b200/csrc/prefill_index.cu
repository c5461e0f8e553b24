// prefill_index.cu -- a3 at prefill: Lightning-Indexer scores of a block of consecutive query
// positions against their causal entries as a tensor-core GEMM.
//
// "Frontier Techniques: NTK RoPE, CSA+HCA, QAT, MTP", 2.1 (the indexer scores every compressed
// entry for every query); the score (reading R3) is s_j = sum_h w_h * relu(q^I_h . K^I_j).  At
// prefill every query of a chunk reads the same keys, so the products run as a GEMM on tcgen05:
// one CTA takes 128 consecutive queries (M) and a range of entries in tiles of 64 (N), with one
// fp32 accumulator per indexer head (K = d_I = 64); the epilogue applies relu and the head
// weights and writes the fp32 scores of each query's causal entries (j < floor(L/m)) row-major, the
// layout the select kernel reads.  No histogram is built here: the select kernel estimates its
// threshold from a sample of the scores (see index_topk.cu).
//
// Warp roles: warp 0 cp.async loader (the CTA's q^I once, then key tiles through a 4-stage ring),
// warp 1 TMEM allocator + MMA issuer, the other warps epilogue, kPsSplit per TMEM lane quarter, each
// over a part of a tile's 64 entries (TMEM -> relu / weights -> shared-memory staging -> coalesced
// row stores).  TMEM holds two accumulator sets (4 heads x 64 columns each)
// so the products of tile t+1 overlap the epilogue of tile t.  Every wait is bounded.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kPsRows = 128;    // queries per CTA (MMA M)
constexpr int kPsTile = 64;     // entries per tile (MMA N)
constexpr int kPsStages = 4;
constexpr int kPsHeads = 4;     // accumulators per tile (H_I <= 4; missing heads get zero rows / weight)
constexpr int kPsSplit = 4;                 // epilogue warps per TMEM lane quarter
constexpr int kPsEpi = 4 * kPsSplit;         // epilogue warps
constexpr int kPsThreads = 64 + 32 * kPsEpi;  // loader, MMA issuer, the epilogue warps
constexpr int kPsPart = kPsTile / kPsSplit;   // entries of a tile one epilogue warp handles
constexpr int kPsStride = kPsPart + 4;        // staging row stride (floats)
static_assert(kPsPart % 16 == 0, "whole 16-column TMEM loads");

struct PsSmem {
    static constexpr int kA = 0;                                    // 4 heads x [128 rows x 128 B]
    static constexpr int kB = kA + kPsHeads * kPsRows * 128;        // stages x [64 rows x 128 B]
    static constexpr int kStg = kB + kPsStages * kPsTile * 128;     // epilogue warps x 32 rows x kPsStride floats
    static constexpr int kBar = kStg + kPsEpi * 32 * kPsStride * 4;
    static constexpr int kMisc = kBar + 16 * 8;
    static constexpr int kTotal = kMisc + 64;
    static constexpr int kAlloc = kTotal + 1024;
};

struct PsBars {
    uint64_t full[kPsStages], empty[kPsStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t a_full, fin;
};

__global__ void __launch_bounds__(kPsThreads, 1) prefill_score_kernel(PrefillScoreParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    PsBars* bars = reinterpret_cast<PsBars*>(sm + PsSmem::kBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + PsSmem::kMisc);  // [0] tmem base, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    const uint32_t sbase = smem_u32(sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    grid_dep_wait();
    grid_dep_launch();
    const int row0 = blockIdx.y * kPsRows;
    const int rows = min(kPsRows, p.Qn - row0);
    // entries visible to the block's last query bound the block's work
    const int64_t e_hi = (p.pos0 + row0 + rows) >> p.m_shift;
    const int64_t e0 = (int64_t)blockIdx.x * p.ent_per_cta;
    if (rows <= 0 || e0 >= e_hi) return;
    const int64_t e1 = min(e_hi, e0 + p.ent_per_cta);
    const int T = (int)((e1 - e0 + kPsTile - 1) / kPsTile);
    const uint16_t* keys = p.entry_keys + p.seq->csa_off * 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kPsStages; ++i) {
            mbar_init(&bars->full[i], 32);
            mbar_init(&bars->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->acc_full[i], 1);
            mbar_init(&bars->acc_empty[i], 32 * kPsEpi);
        }
        mbar_init(&bars->a_full, 32);
        mbar_init(&bars->fin, 1);
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(misc, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        // ------------------------------------------------------------------ loader
        // q^I of the block: head h, row r -> A_h row r (128 bytes, 128-byte swizzle); zero rows past
        // the chunk and for heads >= H_I
        for (int i = lane; i < kPsHeads * kPsRows * 8; i += 32) {
            const int h = i / (kPsRows * 8), r = (i / 8) % kPsRows, c = i % 8;
            const bool ok = r < rows && h < p.H_I;
            const uint16_t* src = ok ? p.q_idx + ((int64_t)(row0 + r) * p.H_I + h) * 64 + c * 8 : p.q_idx;
            cp_async16(sbase + PsSmem::kA + h * kPsRows * 128 + sw128_offset(r, c), src, ok ? 16u : 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(&bars->a_full);
        for (int t = 0; t < T; ++t) {
            const int st = t % kPsStages;
            if (t >= kPsStages && !mbar_wait(&bars->empty[st], ((t / kPsStages) - 1) & 1, p.status, abort_flag)) break;
            const int64_t tb = e0 + (int64_t)t * kPsTile;
            for (int i = lane; i < kPsTile * 8; i += 32) {
                const int r = i / 8, c = i % 8;
                const bool ok = tb + r < e1;
                const uint16_t* src = ok ? keys + (tb + r) * 64 + c * 8 : keys;
                cp_async16(sbase + PsSmem::kB + st * kPsTile * 128 + sw128_offset(r, c), src, ok ? 16u : 0u);
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            mbar_arrive(&bars->full[st]);
        }
        cp_async_wait_all();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        // the whole warp runs the loop (warp-uniform waits and operands); one elected lane issues
        {
            constexpr uint32_t id = idesc_bf16(kPsRows, kPsTile, false, false);
            bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->a_full, 0, p.status, abort_flag));
            for (int t = 0; ok && t < T; ++t) {
                const int st = t % kPsStages, ab = t & 1;
                bool w = mbar_wait(&bars->full[st], (t / kPsStages) & 1, p.status, abort_flag);
                if (w && t >= 2) w = mbar_wait(&bars->acc_empty[ab], ((t >> 1) - 1) & 1, p.status, abort_flag);
                if (!__all_sync(0xffffffffu, w)) break;
                tc_fence_after();
                const uint64_t bd = sdesc_kmajor(sbase + PsSmem::kB + st * kPsTile * 128);
#pragma unroll
                for (int h = 0; h < kPsHeads; ++h) {
                    const uint64_t ad = sdesc_kmajor(sbase + PsSmem::kA + h * kPsRows * 128);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + (uint32_t)(ab * 256 + h * 64), ad + (uint64_t)((ks * 32) >> 4),
                                  bd + (uint64_t)((ks * 32) >> 4), id, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bars->empty[st]);
                umma_commit(&bars->acc_full[ab]);
            }
            umma_commit(&bars->fin);
            mbar_wait(&bars->fin, 0, p.status, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - 2;                 // 0 .. kPsEpi - 1
        const int sp = warp & 3;                 // TMEM sub-partition of this warp: rows 32 sp .. 32 sp + 31
        const int ch = ew >> 2;                  // this warp's part of each tile: entries kPsPart ch .. + kPsPart - 1
        const int r = sp * 32 + lane;            // this lane's query row in the block
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        float wv[kPsHeads];
#pragma unroll
        for (int h = 0; h < kPsHeads; ++h) wv[h] = (r < rows && h < p.H_I) ? p.w[(int64_t)(row0 + r) * p.H_I + h] : 0.f;
        float* stg = reinterpret_cast<float*>(sm + PsSmem::kStg) + ew * 32 * kPsStride;
        // causal entries of this lane's row (the store loop below broadcasts them row by row)
        const int e_mine = (int)((p.pos0 + row0 + r + 1) >> p.m_shift);
        // store loop: kPsPart / 2 lanes per row (two entries each), 64 / kPsPart rows per instruction
        constexpr int kLpr = kPsPart / 2, kRpi = 32 / kLpr;
        const int hl = lane / kLpr, l16 = lane % kLpr;
        for (int t = 0; t < T; ++t) {
            const int ab = t & 1;
            if (!mbar_wait(&bars->acc_full[ab], (t >> 1) & 1, p.status, abort_flag)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kPsPart; c += 16) {
                uint32_t v[kPsHeads][16];
#pragma unroll
                for (int h = 0; h < kPsHeads; ++h)
                    tmem_ld16(tmem + lane_base + (uint32_t)(ab * 256 + h * 64 + ch * kPsPart + c), v[h]);
                tmem_ld_wait();
#pragma unroll
                for (int j4 = 0; j4 < 16; j4 += 4) {
                    float o[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float s = 0.f;
#pragma unroll
                        for (int h = 0; h < kPsHeads; ++h) s = fmaf(wv[h], fmaxf(__uint_as_float(v[h][j4 + j]), 0.f), s);
                        o[j] = s;
                    }
                    *reinterpret_cast<float4*>(stg + lane * kPsStride + c + j4) = make_float4(o[0], o[1], o[2], o[3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty[ab]);
            __syncwarp();
            // the warp's 32 rows, kRpi row parts per instruction (lane: two entries)
            const int64_t tb = e0 + (int64_t)t * kPsTile + ch * kPsPart + 2 * l16;
            for (int rr = 0; rr < 32; rr += kRpi) {
                const int row = sp * 32 + rr + hl;
                const int64_t e_row = __shfl_sync(0xffffffffu, e_mine, rr + hl);  // causal entries of this query
                if (row < rows) {
                    float* dst = p.scores + (int64_t)(row0 + row) * p.e_stride;
                    const float2 v2 = *reinterpret_cast<const float2*>(stg + (rr + hl) * kPsStride + 2 * l16);
                    if (tb + 1 < e_row) *reinterpret_cast<float2*>(dst + tb) = v2;
                    else if (tb < e_row) dst[tb] = v2.x;
                }
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_prefill_scores(const PrefillScoreParams& p, int64_t max_entries, cudaStream_t stream, bool pdl) {
    if (p.Qn <= 0 || max_entries <= 0) return cudaSuccess;
    static PerDeviceOnce attr;
    cudaError_t ea = attr.run([] {
        return cudaFuncSetAttribute(prefill_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PsSmem::kAlloc);
    });
    if (ea != cudaSuccess) return ea;
    const int64_t gx = (max_entries + p.ent_per_cta - 1) / p.ent_per_cta;
    const int64_t gy = (p.Qn + kPsRows - 1) / kPsRows;
    return launch_kernel(prefill_score_kernel, dim3((unsigned)gx, (unsigned)gy), dim3(kPsThreads), PsSmem::kAlloc,
                         stream, pdl, p);
}

}  // namespace csa

// index_topk.cu -- a3/a4: Lightning-Indexer scores and exact top-k.
//
// "Frontier Techniques: NTK RoPE, CSA+HCA, QAT, MTP", 2.1 (the Lightning Indexer scores the
// compressed entries; each query keeps the top-1024); "DeepSeek V4 comprimeix el context: aixi
// funcionen CSA i HCA", "CSA: buscar primer i atendre despres" (a light indexer scores every
// compressed entry and only the best are attended).  Score (reading R3):
//     s_j = sum_h w_h * relu(q^I_h . K^I_j),   j < floor(L / m);
// top-k by (score desc, index asc), written in ascending index order, -1 past the end.
//
// Two kernels:
//  scan   -- grid (chunks, queries).  Streams the indexer-key cache with coalesced 16-byte loads
//            and computes the [16 entries x d_I] . [d_I x H_I] products on the tensor cores
//            (mma.sync m16n8k16, K permuted so that every thread's operand is one contiguous
//            16-byte load), applies relu / head weights in registers, writes the fp32 score and
//            accumulates a coarse histogram of the top 11 bits of the order-preserving score key.
//  select -- grid (filter CTAs, queries).  Every CTA finds the threshold bin from the histogram,
//            sends its entries above it to the result list and those inside it to a candidate
//            list; the last CTA of a query (ticket, no spinning) radix-selects the exact winners
//            among the candidates on the 64-bit key (score key << 32 | ~index), which makes
//            every key unique and breaks ties to the lower index, sorts the k indices and writes
//            them.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kScanThreads = 256;
constexpr int kSelectThreads = 512;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Streaming 16-byte load: not kept in L1, first to be evicted from L2.
__device__ __forceinline__ uint4 ld_stream(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// Scores of 16 consecutive entries (rows r0 .. r0+15 of the key cache) for one warp.
// KV = number of 16-byte vectors per key row (d_I / 8 / 4 per thread group): d_I = 64 -> 2, 32 -> 1.
template <int KV>
__device__ __forceinline__ void score16(const uint16_t* keys, int64_t r0, int64_t nrows, int g, int c,
                                        const uint32_t (&bq)[2 * KV][2], const float (&wv)[2], uint64_t pol,
                                        float& s_lo, float& s_hi) {
    // thread (g, c) loads rows g and g+8, vectors [32*v + 8c, 32*v + 8c + 8) for v < KV
    uint4 lo[KV], hi[KV];
    const int64_t rl = r0 + g, rh = r0 + g + 8;
#pragma unroll
    for (int v = 0; v < KV; ++v) {
        lo[v] = rl < nrows ? ld_stream(keys + rl * (KV * 32) + v * 32 + c * 8, pol) : make_uint4(0, 0, 0, 0);
        hi[v] = rh < nrows ? ld_stream(keys + rh * (KV * 32) + v * 32 + c * 8, pol) : make_uint4(0, 0, 0, 0);
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int v = 0; v < KV; ++v) {
        // k-step 2v uses (x, y), k-step 2v+1 uses (z, w) of the thread's vector
        uint32_t a0[4] = {lo[v].x, hi[v].x, lo[v].y, hi[v].y};
        uint32_t a1[4] = {lo[v].z, hi[v].z, lo[v].w, hi[v].w};
        mma_bf16_16816(acc, a0, bq[2 * v]);
        mma_bf16_16816(acc, a1, bq[2 * v + 1]);
    }
    // acc[0], acc[1]: row g, heads 2c, 2c+1; acc[2], acc[3]: row g+8
    float pl = wv[0] * fmaxf(acc[0], 0.f) + wv[1] * fmaxf(acc[1], 0.f);
    float ph = wv[0] * fmaxf(acc[2], 0.f) + wv[1] * fmaxf(acc[3], 0.f);
    pl += __shfl_xor_sync(0xffffffffu, pl, 1);
    ph += __shfl_xor_sync(0xffffffffu, ph, 1);
    pl += __shfl_xor_sync(0xffffffffu, pl, 2);
    ph += __shfl_xor_sync(0xffffffffu, ph, 2);
    s_lo = pl;
    s_hi = ph;
}

template <int KV>
__global__ void __launch_bounds__(kScanThreads) index_scan_kernel(IndexParams p) {
    __shared__ uint32_t hist[kHistBins];
    __shared__ float sc[kScanThreads / 32][4][16];
    grid_dep_wait();  // the query table may come from the previous kernel
    grid_dep_launch();
    const int qi = blockIdx.y;
    const csa_query qr = p.queries[qi];
    if (qr.seq < 0 || qr.reserved != 0) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const csa_seq sq = p.seqs[qr.seq];
    if (qr.len < 1 || qr.len > sq.len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const int64_t E = qr.len / p.m;
    if (E <= p.k) return;  // everything is selected; the select kernel handles it alone
    if (E > p.max_entries) {  // longer than the grid was sized for: the select kernel reports it
        return;
    }
    const int64_t c0 = (int64_t)blockIdx.x * p.chunk;
    if (c0 >= E) return;
    const int64_t c1 = min(E, c0 + p.chunk);
    for (int i = threadIdx.x; i < kHistBins; i += kScanThreads) hist[i] = 0u;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    // B fragments (query, permuted exactly like the key loads) and head weights
    uint32_t bq[2 * KV][2];
    float wv[2];
    {
        const uint16_t* qrow = p.q_idx + ((int64_t)qi * p.H_I + g) * p.d_I;
        const bool hv = g < p.H_I;
#pragma unroll
        for (int v = 0; v < KV; ++v) {
            uint4 t = hv ? *reinterpret_cast<const uint4*>(qrow + v * 32 + c * 8) : make_uint4(0, 0, 0, 0);
            bq[2 * v][0] = t.x; bq[2 * v][1] = t.y;
            bq[2 * v + 1][0] = t.z; bq[2 * v + 1][1] = t.w;
        }
        const int h0 = 2 * c, h1 = 2 * c + 1;
        wv[0] = h0 < p.H_I ? p.w[(int64_t)qi * p.H_I + h0] : 0.f;
        wv[1] = h1 < p.H_I ? p.w[(int64_t)qi * p.H_I + h1] : 0.f;
    }
    __syncthreads();

    const uint16_t* keys = p.entry_keys + sq.csa_off * p.d_I;
    float* srow = p.scores + (int64_t)qi * p.e_stride;
    const uint64_t pol = policy_evict_first();
    constexpr int kRowsPerPass = kScanThreads / 32 * 16 * 4;  // 512 entries: 4 groups of 16 per warp
    for (int64_t base = c0; base < c1; base += kRowsPerPass) {
        float s[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t r0 = base + (int64_t)(u * (kScanThreads / 32) + warp) * 16;
            score16<KV>(keys, r0, c1, g, c, bq, wv, pol, s[u][0], s[u][1]);
        }
        // stage in shared memory, then coalesced store + histogram
        if (c == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u) { sc[warp][u][g] = s[u][0]; sc[warp][u][g + 8] = s[u][1]; }
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (lane < 16) {
                const int64_t r = base + (int64_t)(u * (kScanThreads / 32) + warp) * 16 + lane;
                if (r < c1) {
                    const float v = sc[warp][u][lane];
                    srow[r] = v;
                    atomicAdd(&hist[float_key(v) >> 21], 1u);
                }
            }
        }
        __syncwarp();
    }
    __syncthreads();
    uint32_t* gh = p.hist + (int64_t)qi * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += kScanThreads)
        if (hist[i]) atomicAdd(&gh[i], hist[i]);
}

// ---- select ----------------------------------------------------------------------------------
//
// One thread-block cluster of F = sel_cluster CTAs per query (1..kSelClusterMax).  CTA c filters the scores of entries
// [c*span, (c+1)*span): every CTA derives the threshold bin from the scan's histogram and keeps the
// entries of that bin and above, as 64-bit keys in index order, in its own shared memory; it then
// publishes its count in the leader CTA (rank 0).  After a cluster barrier every CTA knows its
// offset and pushes its keys into the leader's list through distributed shared memory; after a
// second barrier the leader radix-selects the exact threshold among the bin's members and
// compacts the k indices, ascending.  A list longer than shared memory holds goes through the
// global segment buffer instead, in the same order.

constexpr int kSelPerMax = 64;                           // scores per thread per round
constexpr int kSelBufMax = kSelPerMax * kSelectThreads;  // scores a CTA stages in shared memory per round
constexpr int kStageSmem = 4096;  // kept keys a CTA stages in its own shared memory
constexpr int kListSmem = 8192;   // kept keys the leader holds (in its score buffer, once filtered)

__device__ __forceinline__ uint64_t composite(uint32_t key, int64_t j) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster; orders all earlier memory accesses (shared, distributed
// shared and global) before all later ones at cluster scope.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address in the shared::cluster window of the location `p` (this CTA's shared memory) in CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_u64(uint32_t addr, uint64_t v) {
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// Block-wide suffix sums over kHistBins bins: suf[b] = sum of hist[b' >= b].  Thread t owns bins
// [4*(511-t), 4*(511-t)+4), so a forward scan over threads is a suffix scan over bins.  Also finds
// the unique bin b with suf[b] >= target > suf[b+1] (target >= 1); writes it to out[0] and
// suf[b+1] to out[1] (out[0] = 0xFFFFFFFF if no bin qualifies).  Uses kSelectThreads threads.
__device__ void suffix_find(const uint32_t* hist, uint32_t* suf, uint32_t* warp_tot, uint32_t target,
                            uint32_t* out) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b0 = 4 * (kSelectThreads - 1 - t);
    uint32_t v[4];
    uint32_t s = 0;
#pragma unroll
    for (int i = 3; i >= 0; --i) { s += hist[b0 + i]; v[i] = s; }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    if (t == 0) out[0] = 0xFFFFFFFFu;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = lane < kSelectThreads / 32 ? warp_tot[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane < kSelectThreads / 32) warp_tot[lane] = x;
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? warp_tot[warp - 1] : 0u) + (incl - s);  // bins above b0+3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t here = before + v[i];
        const uint32_t above = i < 3 ? before + v[i + 1] : before;
        suf[b0 + i] = here;
        if (here >= target && above < target) { out[0] = (uint32_t)(b0 + i); out[1] = above; }
    }
    __syncthreads();
}

// Block-wide exclusive scan of one value per thread; returns this thread's exclusive prefix and
// writes the total to *total.  `wsum` holds kSelectThreads/32 words.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = lane < kSelectThreads / 32 ? wsum[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane < kSelectThreads / 32) wsum[lane] = x;
    }
    __syncthreads();
    const uint32_t excl = (warp > 0 ? wsum[warp - 1] : 0u) + incl - v;
    *total = wsum[kSelectThreads / 32 - 1];
    __syncthreads();
    return excl;
}

// The kept list of one query: the cluster CTAs' key runs concatenated in rank order (so in index
// order), either gathered in the leader's shared memory (`cache`) or left in the global segment
// buffer, where run c starts at seg + c*span and entry i lives in the last run c with off[c] <= i.
struct KeptList {
    const uint64_t* seg;
    const uint32_t* off;     // [F + 1] exclusive prefix of the run lengths
    int F;                   // CTAs in the cluster
    int64_t span;
    const uint64_t* cache;
    __device__ __forceinline__ uint64_t get(uint32_t i) const {
        if (cache) return cache[i];
        int c = 0;
        for (int r = 1; r < F; ++r) c += off[r] <= i ? 1 : 0;
        return __ldcg(reinterpret_cast<const unsigned long long*>(seg) + (int64_t)c * span + (i - off[c]));
    }
};

// Exact selection of the `need` largest keys among the list entries whose top 11 bits equal top11
// (the threshold-bin members; entries of higher bins are kept regardless).  Returns T with exactly
// `need` of those members >= T.  Radix passes of 11 bits over bits 52..0, counted with
// shared-memory atomics; stops as soon as the chosen digit holds exactly the remaining count.
__device__ uint64_t radix_threshold(const KeptList& L, uint32_t n, uint32_t need, uint32_t top11, uint32_t* cnt,
                                    uint32_t* suf, uint32_t* misc) {
    uint64_t prefix = (uint64_t)top11 << 53;
    uint64_t mask = (uint64_t)0x7FF << 53;
    uint32_t remaining = need;
    for (int shift = 42;; shift -= 11) {
        const int sh = shift < 0 ? 0 : shift;
        const int bits = shift < 0 ? 11 + shift : 11;
        const uint32_t dmask = (1u << bits) - 1u;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) cnt[i] = 0;
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < n; i += blockDim.x) {
            const uint64_t v = L.get(i);
            if ((v & mask) == prefix) atomicAdd(&cnt[(uint32_t)(v >> sh) & dmask], 1u);
        }
        __syncthreads();
        suffix_find(cnt, suf, misc, remaining, misc + 48);  // misc[0..15]: warp totals
        const uint32_t dg = misc[48];
        const uint32_t above = misc[49];
        const uint32_t in_digit = cnt[dg];
        __syncthreads();
        remaining -= above;
        prefix |= (uint64_t)dg << sh;
        mask |= (uint64_t)dmask << sh;
        if (in_digit == remaining || sh == 0) return prefix;  // lower bits left at zero
    }
}

// Dynamic shared memory of the select kernel.
struct SelSmem {
    static constexpr int kHist = 0;                          // u32[kHistBins]
    static constexpr int kSuf = kHist + kHistBins * 4;       // u32[kHistBins]
    static constexpr int kMisc = kSuf + kHistBins * 4;       // u32[64]
    static constexpr int kXcnt = kMisc + 64 * 4;             // u32[32]: the leader's run lengths (| overflow bit)
    static constexpr int kOffs = kXcnt + 32 * 4;             // u32[32]: exclusive prefix, F + 1 used
    static constexpr int kStage = kOffs + 32 * 4;            // u64[kStageSmem]: this CTA's run
    static constexpr int kBuf = kStage + kStageSmem * 8;     // f32[sel_buf] scores; the leader's list
                                                             // (u64[kListSmem]) once it has filtered
    // dynamic shared memory of a launch staging `buf` scores per round
    static constexpr size_t bytes(int64_t buf) {
        return (size_t)kBuf + (buf * 4 > (int64_t)kListSmem * 8 ? (size_t)buf * 4 : (size_t)kListSmem * 8);
    }
};

__global__ void __launch_bounds__(kSelectThreads) index_select_kernel(IndexParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw + SelSmem::kHist);
    uint32_t* suf = reinterpret_cast<uint32_t*>(smem_raw + SelSmem::kSuf);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + SelSmem::kMisc);
    uint32_t* xcnt = reinterpret_cast<uint32_t*>(smem_raw + SelSmem::kXcnt);
    uint32_t* offs = reinterpret_cast<uint32_t*>(smem_raw + SelSmem::kOffs);
    uint64_t* stage = reinterpret_cast<uint64_t*>(smem_raw + SelSmem::kStage);
    uint64_t* lst = reinterpret_cast<uint64_t*>(smem_raw + SelSmem::kBuf);
    __shared__ uint32_t s_wsum[kSelectThreads / 32];
    __shared__ uint64_t s_bar;
    __shared__ int s_abort;
    grid_dep_wait();  // scores and histogram come from the scan kernel
    grid_dep_launch();

    // Every branch below that returns before the cluster barriers depends only on the query, so all
    // CTAs of a cluster take it together.
    const int qi = blockIdx.y;
    const uint32_t rank = cluster_rank();
    const csa_query qr = p.queries[qi];
    const bool seq_ok = qr.seq >= 0 && qr.reserved == 0;
    const csa_seq sq = seq_ok ? p.seqs[qr.seq] : csa_seq{0, 0, 0, 0};
    const bool valid = seq_ok && qr.len >= 1 && qr.len <= sq.len;
    int64_t E = valid ? qr.len / p.m : 0;
    if (E > p.max_entries || !seq_ok) {  // the launch was sized for fewer entries: refuse rather than guess
        if (threadIdx.x == 0 && rank == 0) report(p.status, CSA_ERR_INDEX);
        E = 0;
    }
    int32_t* out = p.idx_out + (int64_t)qi * p.k;
    float* sout = p.score_out ? p.score_out + (int64_t)qi * p.k : nullptr;
    const float* srow = p.scores + (int64_t)qi * p.e_stride;

    if (E <= p.k) {  // select everything: no scores were computed
        if (rank != 0) return;
        for (int i = threadIdx.x; i < p.k; i += blockDim.x) {
            out[i] = i < E ? i : -1;
            if (sout) sout[i] = __int_as_float(0x7FC00000);
        }
        if (sout && E > 0) {
            // scores of the selected entries (recomputed here; E <= k is small)
            for (int64_t j = threadIdx.x; j < E; j += blockDim.x) {
                const uint16_t* kr = p.entry_keys + (sq.csa_off + j) * p.d_I;
                float s = 0.f;
                for (int h = 0; h < p.H_I; ++h) {
                    const uint16_t* qh = p.q_idx + ((int64_t)qi * p.H_I + h) * p.d_I;
                    float dot = 0.f;
                    for (int cc = 0; cc < p.d_I; ++cc)
                        dot = fmaf(__uint_as_float((uint32_t)qh[cc] << 16), __uint_as_float((uint32_t)kr[cc] << 16), dot);
                    s += p.w[(int64_t)qi * p.H_I + h] * fmaxf(dot, 0.f);
                }
                sout[j] = s;
            }
        }
        return;
    }

    const int F = p.sel_cluster;
    const int64_t c0 = (int64_t)rank * p.sel_span;
    const int64_t c1 = min(E, c0 + p.sel_span);
    // Rounds of sel_buf scores are staged in shared memory by bulk copies (the first round's copy
    // goes out before the histogram loads).
    float* sbuf = reinterpret_cast<float*>(smem_raw + SelSmem::kBuf);
    const uint32_t sbuf_addr = smem_u32(sbuf);
    const int lane = threadIdx.x & 31;
    const int L = p.sel_per;  // entries per thread per round: a power of two, 4..kSelPerMax
    const int G = L / 4;
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    __syncthreads();
    // thread 0: copy the 16-byte-multiple part of round [rb, rb + n) into sbuf
    auto issue_round = [&](int64_t rb) {
        const int64_t n = min((int64_t)p.sel_buf, c1 - rb);
        const uint32_t bytes = (uint32_t)(n & ~(int64_t)3) * 4u;
        fence_proxy_async_smem();  // earlier generic accesses to sbuf come first
        if (bytes == 0) {
            mbar_arrive(&s_bar);
            return;
        }
        mbar_arrive_expect_tx(&s_bar, bytes);
        for (uint32_t off = 0; off < bytes; off += 65536u)
            bulk_load(sbuf_addr + off, srow + rb + off / 4u, min(65536u, bytes - off), &s_bar);
    };
    if (threadIdx.x == 0 && c0 < c1) issue_round(c0);

    uint64_t* gseg = p.seg + (int64_t)qi * p.e_seg + (int64_t)rank * p.sel_span;
    uint32_t n_mine = 0;
    bool spilled = false;  // the run lives in gseg instead of `stage`
    bool failed = false;
    // Keep the entries of [rb, rb + n) (staged in sbuf) whose bin is >= b_lo, appending them in
    // index order to the run.  Thread t filters entries [t*L, t*L + L), reading its float4 groups in
    // an order rotated by the lane so a warp's reads spread over all banks; bit 4*g + e of m64 flags
    // entry 4*g + e of the thread's range.
    auto filter_round = [&](int64_t rb, int64_t n, uint32_t b_lo) {
        const float thr = key_float(b_lo << 21);  // the smallest float of bin b_lo (b_lo = 0: keep all)
        const bool keep_all = b_lo == 0u;
        const int64_t tb = (int64_t)threadIdx.x * L;
        const int64_t valid = n - tb < 0 ? 0 : (n - tb > L ? L : n - tb);
        uint64_t m64 = 0;
        if (!failed && valid > 0) {
            const float4* s4 = reinterpret_cast<const float4*>(sbuf + tb);
#pragma unroll 4
            for (int g = 0; g < G; ++g) {
                const int gg = (g + lane) & (G - 1);
                const float4 v = s4[gg];
                // a float compare against the bin's lower edge passes every kept entry (the key is
                // monotone in the float order); passes are confirmed on the exact key below, which
                // also drops -0.0 below a +0.0 edge
                const uint32_t m = keep_all ? 0xFu
                                            : (v.x >= thr ? 1u : 0u) | (v.y >= thr ? 2u : 0u) |
                                                  (v.z >= thr ? 4u : 0u) | (v.w >= thr ? 8u : 0u);
                m64 |= (uint64_t)m << (4 * gg);
            }
            if (valid < 64) m64 &= (1ull << valid) - 1ull;
            for (uint64_t c = m64; c; c &= c - 1ull) {
                const int bit = __ffsll((long long)c) - 1;
                if ((float_key(sbuf[tb + bit]) >> 21) < b_lo) m64 &= ~(1ull << bit);
            }
        }
        uint32_t tot;
        uint32_t pos = block_excl_scan((uint32_t)__popcll(m64), s_wsum, &tot);
        if (!spilled && n_mine + tot > (uint32_t)kStageSmem) {
            for (uint32_t i = threadIdx.x; i < n_mine; i += blockDim.x) gseg[i] = stage[i];
            spilled = true;
            __syncthreads();
        }
        pos += n_mine;
        for (; m64; m64 &= m64 - 1ull) {
            const int bit = __ffsll((long long)m64) - 1;
            const uint64_t key = composite(float_key(sbuf[tb + bit]), rb + tb + bit);
            if (spilled) gseg[pos] = key;
            else stage[pos] = key;
            ++pos;
        }
        n_mine += tot;
        __syncthreads();
    };

    uint32_t b1, above, need, n_bin;
    if (!p.sampled) {
        // 1. threshold bin from the scan's histogram (every CTA of the query finds the same one)
        const uint32_t* gh = p.hist + (int64_t)qi * kHistBins;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = __ldcg(gh + i);
        __syncthreads();
        suffix_find(hist, suf, misc, (uint32_t)p.k, misc + 32);
        b1 = misc[32];
        above = misc[33];
        need = (uint32_t)p.k - above;
        n_bin = b1 == 0xFFFFFFFFu ? 0u : hist[b1];  // members of the threshold bin
        failed = b1 == 0xFFFFFFFFu;                 // histogram holds fewer than k scores: cannot happen

        // 2. keep this CTA's entries of bin >= b1, in index order, round by round
        uint32_t phase = 0;
        for (int64_t rb = c0; rb < c1; rb += p.sel_buf) {
            const int64_t n = min((int64_t)p.sel_buf, c1 - rb);
            const int64_t n16 = n & ~(int64_t)3;
            if (threadIdx.x < n - n16) sbuf[n16 + threadIdx.x] = __ldg(srow + rb + n16 + threadIdx.x);
            // a wait that runs out leaves this CTA's run empty (and the status word set); the CTA
            // still takes both cluster barriers below
            if (!mbar_wait(&s_bar, phase, p.status, &s_abort)) failed = true;
            phase ^= 1u;
            __syncthreads();
            filter_round(rb, n, b1);  // ends with a barrier: sbuf is free again
            if (threadIdx.x == 0 && rb + p.sel_buf < c1) issue_round(rb + p.sel_buf);
        }
    } else {
        // No histogram (prefill GEMM scores; one CTA holds the query's whole row in one round).
        // 1'. estimate a bin from a sample: the bin below which about 2k / n of the sample lies is
        //     low enough that at least k entries pass it with overwhelming probability
        const int64_t n = c1 - c0;
        const int64_t n16 = n & ~(int64_t)3;
        if (threadIdx.x < n - n16) sbuf[n16 + threadIdx.x] = __ldg(srow + c0 + n16 + threadIdx.x);
        if (n > 0 && !mbar_wait(&s_bar, 0, p.status, &s_abort)) failed = true;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        const int64_t S = n < 4096 ? n : 4096;
        for (int64_t i = threadIdx.x; i < S; i += blockDim.x)
            atomicAdd(&hist[float_key(sbuf[(i * n) / S]) >> 21], 1u);
        __syncthreads();
        const int64_t want = (2 * (int64_t)p.k * S + n - 1) / (n > 0 ? n : 1);
        suffix_find(hist, suf, misc, (uint32_t)(want < S ? want : S + 1), misc + 32);
        uint32_t b_est = misc[32] == 0xFFFFFFFFu ? 0u : misc[32];  // no bin qualifies: keep everything
        // 2'. candidates: every entry of bin >= b_est, in index order
        filter_round(c0, n, b_est);
        if (n_mine < (uint32_t)p.k && b_est > 0) {  // the estimate was too high (rare): keep everything
            n_mine = 0;
            spilled = false;
            filter_round(c0, n, 0u);
        }
        // 3'. the exact threshold bin from the candidates' own histogram
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < n_mine; i += blockDim.x) {
            const uint64_t key = spilled ? __ldcg(reinterpret_cast<const unsigned long long*>(gseg) + i) : stage[i];
            atomicAdd(&hist[(uint32_t)(key >> 53)], 1u);
        }
        __syncthreads();
        suffix_find(hist, suf, misc, (uint32_t)p.k, misc + 32);
        b1 = misc[32];
        above = misc[33];
        need = (uint32_t)p.k - above;
        n_bin = b1 == 0xFFFFFFFFu ? 0u : hist[b1];
        if (b1 == 0xFFFFFFFFu) failed = true;
    }
    if (failed) n_mine = 0;

    // 3. run lengths to the leader, then every CTA learns its offset
    if (threadIdx.x == 0) st_cluster_u32(map_rank(&xcnt[rank], 0), n_mine | (spilled ? 0x80000000u : 0u));
    cluster_sync();
    if (threadIdx.x < F) suf[threadIdx.x] = ld_cluster_u32(map_rank(&xcnt[threadIdx.x], 0));
    __syncthreads();
    uint32_t off_me = 0, total = 0;
    bool any_spill = false;
    for (int c = 0; c < F; ++c) {
        const uint32_t v = suf[c];
        if ((uint32_t)c < rank) off_me += v & 0x7FFFFFFFu;
        if (threadIdx.x == 0) offs[c] = total;
        total += v & 0x7FFFFFFFu;
        any_spill |= (v >> 31) != 0u;
    }
    if (threadIdx.x == 0) offs[F] = total;
    // every CTA has read the histogram: clear it for the next call, one share per CTA
    {
        uint32_t* ghw = p.hist + (int64_t)qi * kHistBins;
        const int share = kHistBins / F;
        for (int i = threadIdx.x; i < share; i += blockDim.x) ghw[rank * share + i] = 0u;
    }
    const bool in_smem = !any_spill && total <= (uint32_t)kListSmem;
    if (in_smem) {
        // the leader's score buffer is free (its filter is done, no copy in flight): it becomes the list
        const uint32_t dst = map_rank(lst + off_me, 0);
        for (uint32_t i = threadIdx.x; i < n_mine; i += blockDim.x) st_cluster_u64(dst + i * 8u, stage[i]);
    } else if (!spilled) {
        for (uint32_t i = threadIdx.x; i < n_mine; i += blockDim.x) gseg[i] = stage[i];
    }
    cluster_sync();
    if (rank != 0) return;

    // 4. the leader: exact threshold, then compaction in index order
    const uint32_t n_tot = total;
    // without sampling the kept list is exactly the entries of bins >= b1; with it, a superset
    if (b1 == 0xFFFFFFFFu || (p.sampled ? n_tot < above + n_bin : n_tot != above + n_bin)) {
        if (threadIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const KeptList kl{p.seg + (int64_t)qi * p.e_seg, offs, F, p.sel_span, in_smem ? lst : nullptr};
    const uint64_t T = need == n_bin ? ((uint64_t)b1 << 53) : radix_threshold(kl, n_tot, need, b1, hist, suf, misc);
    const uint32_t per_t = (n_tot + blockDim.x - 1) / blockDim.x;
    const uint32_t i0 = threadIdx.x * per_t, i1 = min(n_tot, i0 + per_t);
    uint32_t mine = 0;
    for (uint32_t i = i0; i < i1; ++i) mine += kl.get(i) >= T ? 1u : 0u;
    uint32_t kept_total;
    uint32_t o = block_excl_scan(mine, s_wsum, &kept_total);
    for (uint32_t i = i0; i < i1; ++i) {
        const uint64_t v = kl.get(i);
        if (v >= T) {
            if (o < (uint32_t)p.k) {
                out[o] = (int32_t)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
                if (sout) sout[o] = key_float((uint32_t)(v >> 32));
            }
            ++o;
        }
    }
    if (threadIdx.x == 0 && kept_total != (uint32_t)p.k) report(p.status, CSA_ERR_INDEX);
}

constexpr size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

cudaError_t select_attrs() {
    static PerDeviceOnce attr;
    return attr.run([] {
        cudaError_t e = cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SelSmem::bytes(kSelBufMax));
        if (e != cudaSuccess) return e;
        return cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
}

size_t index_ws_bytes(int Q, int64_t e_stride) {
    size_t s = 0;
    s += align256((size_t)Q * kHistBins * 4);
    s += align256((size_t)Q * e_stride * 4);
    s += align256((size_t)Q * (e_stride + 8 * kSelClusterMax) * 8);
    return s;
}

size_t index_zero_bytes(int Q) { return align256((size_t)Q * kHistBins * 4); }

void index_ws_carve(IndexParams& p, void* ws, int Q, int64_t e_stride) {
    char* b = static_cast<char*>(ws);
    p.hist = reinterpret_cast<uint32_t*>(b);
    b += align256((size_t)Q * kHistBins * 4);
    p.scores = reinterpret_cast<float*>(b);
    b += align256((size_t)Q * e_stride * 4);
    p.seg = reinterpret_cast<uint64_t*>(b);
    p.e_stride = e_stride;
    p.e_seg = e_stride + 8 * kSelClusterMax;
}

cudaError_t launch_index_topk(IndexParams& p, int64_t max_entries, cudaStream_t stream, bool zero_ws,
                              cudaEvent_t mid, bool pdl, bool sampled) {
    p.sampled = sampled ? 1 : 0;
    if (sampled) {
        // scores are already in p.scores; one select CTA per query holds its whole row
        if (max_entries > kSelBufMax) return cudaErrorInvalidValue;
        p.sel_cluster = 1;
        p.sel_span = ((max_entries + 7) / 8) * 8;
        if (p.sel_span < 8) p.sel_span = 8;
        int per = 4;
        while (per < kSelPerMax && (int64_t)per * kSelectThreads < p.sel_span) per *= 2;
        p.sel_per = per;
        p.sel_buf = per * kSelectThreads;
        const size_t smem = SelSmem::bytes(p.sel_buf);
        cudaError_t e = select_attrs();
        if (e != cudaSuccess) return e;
        return launch_kernel_cluster(index_select_kernel, dim3(1, (unsigned)p.Q), dim3(kSelectThreads), smem, stream,
                                     pdl, dim3(1, 1, 1), p);
    }
    if (zero_ws) {
        // the histogram sits at the start of the workspace
        cudaError_t e = cudaMemsetAsync(p.hist, 0, index_zero_bytes(p.Q), stream);
        if (e != cudaSuccess) return e;
    }
    if (max_entries > p.k) {
        const int64_t total = max_entries * (int64_t)p.Q;
        // aim for ~4 scan CTAs per SM over all queries, chunks of 512..16384 entries
        int64_t chunk = (total + 148 * 4 - 1) / (148 * 4);
        chunk = ((chunk + 511) / 512) * 512;
        if (chunk < 512) chunk = 512;
        if (chunk > 16384) chunk = 16384;
        p.chunk = chunk;
        const int64_t gx = (max_entries + chunk - 1) / chunk;
        cudaError_t e = p.d_I == 64
                            ? launch_kernel(index_scan_kernel<2>, dim3((unsigned)gx, (unsigned)p.Q), dim3(kScanThreads), 0,
                                            stream, pdl && !zero_ws, p)
                            : launch_kernel(index_scan_kernel<1>, dim3((unsigned)gx, (unsigned)p.Q), dim3(kScanThreads), 0,
                                            stream, pdl && !zero_ws, p);
        if (e != cudaSuccess) return e;
    }
    if (mid) {
        cudaError_t e = cudaEventRecordWithFlags(mid, stream, cudaEventRecordExternal);
        if (e != cudaSuccess) return e;
    }
    // cluster size: about two select CTAs per SM over all queries, 1..kSelClusterMax CTAs per query
    int F = 1;
    while (F < kSelClusterMax && (int64_t)p.Q * F * 2 <= 2 * 148) F *= 2;
    p.sel_cluster = F;
    p.sel_span = (((p.e_stride + F - 1) / F + 7) / 8) * 8;  // F * span <= e_stride + 8F <= e_seg
    // scores per thread per round: the smallest power of two that covers the CTA's span in one
    // round, 4..kSelPerMax; the round buffer holds that many per thread
    int per = 4;
    while (per < kSelPerMax && (int64_t)per * kSelectThreads < p.sel_span) per *= 2;
    p.sel_per = per;
    p.sel_buf = per * kSelectThreads;
    const int64_t buf = p.sel_buf;
    const size_t smem = SelSmem::bytes(buf);
    cudaError_t ea = select_attrs();
    if (ea != cudaSuccess) return ea;
    // after an event record the select follows the scan without overlap
    return launch_kernel_cluster(index_select_kernel, dim3((unsigned)F, (unsigned)p.Q), dim3(kSelectThreads), smem,
                                 stream, pdl && mid == nullptr, dim3((unsigned)F, 1, 1), p);
}

}  // namespace csa

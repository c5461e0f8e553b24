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

constexpr int kSelPerThread = kSelPerCta / kSelectThreads;          // 8 scores per thread
constexpr int kListSmem = 8192;                                     // kept entries the last CTA holds

__device__ __forceinline__ uint64_t composite(uint32_t key, int64_t j) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
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

// The kept list of one query: the filter CTAs' segments concatenated in CTA order (so in index
// order).  Entry i lives in segment c = the last with off[c] <= i.
struct KeptList {
    const uint64_t* seg;     // [F][kSelPerCta]
    const uint32_t* off;     // [F + 1] exclusive prefix of the segment counts (shared memory)
    int F;
    const uint64_t* cache;   // the whole list in shared memory, or nullptr
    __device__ __forceinline__ uint64_t get(uint32_t i) const {
        if (cache) return cache[i];
        int lo = 0, hi = F - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off[mid] <= i) lo = mid; else hi = mid - 1;
        }
        return __ldcg(reinterpret_cast<const unsigned long long*>(seg) + (int64_t)lo * kSelPerCta + (i - off[lo]));
    }
};

// Exact selection of the `need` largest keys among the list entries whose top 11 bits equal top11
// (the threshold-bin members; entries of higher bins are kept regardless).  Returns T with exactly
// `need` of those members >= T.  Radix passes of 11 bits over bits 52..0 (counted with
// warp-aggregated shared-memory atomics, so equal digits do not serialize); stops as soon as the
// chosen digit holds exactly the remaining count.
__device__ uint64_t radix_threshold(const KeptList& L, uint32_t n, uint32_t need, uint32_t top11, uint32_t* cnt,
                                    uint32_t* suf, uint32_t* misc) {
    uint64_t prefix = (uint64_t)top11 << 53;
    uint64_t mask = (uint64_t)0x7FF << 53;
    uint32_t remaining = need;
    const int lane = threadIdx.x & 31;
    for (int shift = 42;; shift -= 11) {
        const int sh = shift < 0 ? 0 : shift;
        const int bits = shift < 0 ? 11 + shift : 11;
        const uint32_t dmask = (1u << bits) - 1u;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) cnt[i] = 0;
        __syncthreads();
        const uint32_t n_round = (n + 31u) & ~31u;
        for (uint32_t i = threadIdx.x; i < n_round; i += blockDim.x) {
            bool match = false;
            uint32_t dg = 0;
            if (i < n) {
                const uint64_t v = L.get(i);
                match = (v & mask) == prefix;
                dg = (uint32_t)(v >> sh) & dmask;
            }
            const uint32_t active = __ballot_sync(0xffffffffu, match);
            if (match) {
                const uint32_t peers = __match_any_sync(active, dg);
                if (lane == __ffs(peers) - 1) atomicAdd(&cnt[dg], (uint32_t)__popc(peers));
            }
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

__global__ void __launch_bounds__(kSelectThreads) index_select_kernel(IndexParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);          // kHistBins
    uint32_t* suf = hist + kHistBins;                                  // kHistBins
    uint32_t* misc = suf + kHistBins;                                  // 64
    uint64_t* lst = reinterpret_cast<uint64_t*>(misc + 64);            // kListSmem
    uint32_t* offs = reinterpret_cast<uint32_t*>(lst + kListSmem);    // filter CTAs + 1
    __shared__ uint32_t s_last;
    __shared__ uint32_t s_wsum[kSelectThreads / 32];
    grid_dep_wait();  // scores and histogram come from the scan kernel
    grid_dep_launch();

    const int qi = blockIdx.y;
    const csa_query qr = p.queries[qi];
    const csa_seq sq = p.seqs[qr.seq];
    const bool valid = qr.len >= 1 && qr.len <= sq.len;
    int64_t E = valid ? qr.len / p.m : 0;
    if (E > p.max_entries) {  // the grid was sized for fewer entries: refuse rather than guess
        if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        E = 0;
    }
    int32_t* out = p.idx_out + (int64_t)qi * p.k;
    float* sout = p.score_out ? p.score_out + (int64_t)qi * p.k : nullptr;
    const float* srow = p.scores + (int64_t)qi * p.e_stride;

    if (E <= p.k) {  // select everything: no scores were computed
        if (blockIdx.x != 0) return;
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

    // 1. threshold bin (every CTA of the query finds the same one)
    const uint32_t* gh = p.hist + (int64_t)qi * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = __ldcg(gh + i);
    __syncthreads();
    suffix_find(hist, suf, misc, (uint32_t)p.k, misc + 32);
    const uint32_t b1 = misc[32];
    const uint32_t above = misc[33];
    if (b1 == 0xFFFFFFFFu) {  // histogram holds fewer than k scores: cannot happen
        if (threadIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const uint32_t need = (uint32_t)p.k - above;
    const uint32_t n_bin = hist[b1];  // members of the threshold bin (over all CTAs)

    // 2. keep this CTA's entries of bin >= b1, in index order, in its own segment
    const int64_t j0 = (int64_t)blockIdx.x * kSelPerCta + (int64_t)threadIdx.x * kSelPerThread;
    float sv[kSelPerThread];
    if (j0 + kSelPerThread <= E) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(srow + j0));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(srow + j0 + 4));
        sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w; sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
    } else {
#pragma unroll
        for (int u = 0; u < kSelPerThread; ++u) sv[u] = j0 + u < E ? __ldcg(srow + j0 + u) : 0.f;
    }
    uint32_t nk = 0, kf = 0;
#pragma unroll
    for (int u = 0; u < kSelPerThread; ++u) {
        if (j0 + u < E && (float_key(sv[u]) >> 21) >= b1) { ++nk; kf |= 1u << u; }
    }
    uint32_t cta_total;
    uint32_t pos = block_excl_scan(nk, s_wsum, &cta_total);
    uint64_t* myseg = p.seg + (int64_t)qi * p.e_seg + (int64_t)blockIdx.x * kSelPerCta;
#pragma unroll
    for (int u = 0; u < kSelPerThread; ++u)
        if (kf & (1u << u)) myseg[pos++] = composite(float_key(sv[u]), j0 + u);
    if (threadIdx.x == 0) p.seg_count[(int64_t)qi * (p.e_seg / kSelPerCta) + blockIdx.x] = cta_total;

    // 3. the last CTA of this query finishes the selection
    uint32_t* ctr = p.counters + (int64_t)qi * 4;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&ctr[0], 1u) == gridDim.x - 1) ? 1u : 0u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int F = gridDim.x;
    // exclusive prefix of the segment counts (8 per thread)
    {
        const uint32_t* gc = p.seg_count + (int64_t)qi * (p.e_seg / kSelPerCta);
        uint32_t c8[8], tot = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = threadIdx.x * 8 + u;
            c8[u] = c < F ? __ldcg(gc + c) : 0u;
            tot += c8[u];
        }
        uint32_t all;
        uint32_t run = block_excl_scan(tot, s_wsum, &all);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = threadIdx.x * 8 + u;
            if (c <= F) offs[c] = run;
            run += c8[u];
        }
        __syncthreads();
    }
    const uint32_t n_tot = offs[F];
    if (n_tot != above + n_bin) {  // histogram and filter disagree: cannot happen
        if (threadIdx.x == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    KeptList kl{p.seg + (int64_t)qi * p.e_seg, offs, F, nullptr};
    if (n_tot <= (uint32_t)kListSmem) {
        for (uint32_t i = threadIdx.x; i < n_tot; i += blockDim.x) lst[i] = kl.get(i);
        __syncthreads();
        kl.cache = lst;
    }
    const uint64_t T = need == n_bin ? ((uint64_t)b1 << 53) : radix_threshold(kl, n_tot, need, b1, hist, suf, misc);
    // 4. compaction in index order: keep every entry >= T (exactly k of them)
    const uint32_t per = (n_tot + blockDim.x - 1) / blockDim.x;
    const uint32_t i0 = threadIdx.x * per, i1 = min(n_tot, i0 + per);
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
    // leave the per-query histogram and ticket clean for the next call
    uint32_t* ghw = p.hist + (int64_t)qi * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ghw[i] = 0u;
    if (threadIdx.x < 4) ctr[threadIdx.x] = 0u;
}

constexpr size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

int64_t seg_stride(int64_t e_stride) { return ((e_stride + kSelPerCta - 1) / kSelPerCta) * kSelPerCta; }

size_t index_ws_bytes(int Q, int64_t e_stride) {
    const int64_t es = seg_stride(e_stride);
    size_t s = 0;
    s += align256((size_t)Q * kHistBins * 4);
    s += align256((size_t)Q * 4 * 4);
    s += align256((size_t)Q * (es / kSelPerCta) * 4);
    s += align256((size_t)Q * e_stride * 4);
    s += align256((size_t)Q * es * 8);
    return s;
}

size_t index_zero_bytes(int Q) { return align256((size_t)Q * kHistBins * 4) + align256((size_t)Q * 4 * 4); }

void index_ws_carve(IndexParams& p, void* ws, int Q, int64_t e_stride) {
    const int64_t es = seg_stride(e_stride);
    char* b = static_cast<char*>(ws);
    p.hist = reinterpret_cast<uint32_t*>(b);
    b += align256((size_t)Q * kHistBins * 4);
    p.counters = reinterpret_cast<uint32_t*>(b);
    b += align256((size_t)Q * 4 * 4);
    p.seg_count = reinterpret_cast<uint32_t*>(b);
    b += align256((size_t)Q * (es / kSelPerCta) * 4);
    p.scores = reinterpret_cast<float*>(b);
    b += align256((size_t)Q * e_stride * 4);
    p.seg = reinterpret_cast<uint64_t*>(b);
    p.e_stride = e_stride;
    p.e_seg = es;
}

cudaError_t launch_index_topk(IndexParams& p, int64_t max_entries, cudaStream_t stream, bool zero_ws,
                              cudaEvent_t mid, bool pdl) {
    if (zero_ws) {
        // histogram + counters are contiguous at the start of the workspace
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
    int64_t f = (max_entries + kSelPerCta - 1) / kSelPerCta;
    if (f < 1) f = 1;
    p.filter_ctas = (int)f;
    if (f > (int64_t)kSelectThreads * 8 - 1) return cudaErrorInvalidValue;  // > 16M entries per query
    const size_t smem = (size_t)kHistBins * 8 + 64 * 4 + (size_t)kListSmem * 8 + ((size_t)f + 1) * 4;
    static bool attr_set = false;
    if (!attr_set) {
        const int max_smem = kHistBins * 8 + 64 * 4 + kListSmem * 8 + kSelectThreads * 8 * 4;
        cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        attr_set = true;
    }
    // after an event record the select follows the scan without overlap
    return launch_kernel(index_select_kernel, dim3((unsigned)f, (unsigned)p.Q), dim3(kSelectThreads), smem, stream,
                         pdl && mid == nullptr, p);
}

}  // namespace csa

// index_topk.cu -- a3/a4: Lightning-Indexer scores and exact top-k.
//
// "Frontier Techniques: NTK RoPE, CSA+HCA, QAT, MTP", 2.1 (the Lightning Indexer scores the
// compressed entries; each query keeps the top-1024); "DeepSeek V4 comprimeix el context: aixi
// funcionen CSA i HCA", "CSA: buscar primer i atendre despres" (a light indexer scores every
// compressed entry and only the best are attended).  Score (reading R3):
//     s_j = sum_h w_h * relu(q^I_h . K^I_j),   j < floor(L / m);
// top-k by (score desc, index asc), written in ascending index order, -1 past the end.  Every
// selection works on the 64-bit key (order-preserving score key << 32 | ~index), which is unique
// and breaks ties to the lower index.
//
// Three kernels:
//  index_scan_kernel   -- grid (chunks, queries), the decode / standalone path.  Streams the
//            indexer-key cache with coalesced 16-byte loads and computes the [16 entries x d_I] .
//            [d_I x H_I] products on the tensor cores (mma.sync m16n8k16, K permuted so that every
//            thread's operand is one contiguous 16-byte load), applies relu / head weights in
//            registers, and counts the scores into the query's histogram of the top kKeyBits key
//            bits.  Each chunk keeps its local candidates.
//  index_final_kernel  -- one thread-block cluster per query after the scan: the exact top-k from
//            the chunks' candidates (see the kernel).
//  index_select_kernel -- one CTA per query, the prefill path: the top-k of a score row that the
//            prefill GEMM stored, with a threshold bin estimated from a sample of the row.
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

// Scores of 16 consecutive entries (rows r0 .. r0+15 of the key cache) for one warp, in two halves:
// load16 issues the loads, score16 forms the scores from them.  A pass issues the loads of all its
// groups before it scores any: an mma waits for its operands, and the loads of the next group must
// not wait behind it.
// KV = number of 16-byte vectors per key row (d_I / 8 / 4 per thread group): d_I = 64 -> 2, 32 -> 1.
template <int KV>
__device__ __forceinline__ void load16(const uint16_t* keys, int64_t r0, int64_t nrows, int g, int c, uint64_t pol,
                                       uint4 (&lo)[KV], uint4 (&hi)[KV]) {
    // thread (g, c) loads rows g and g+8, vectors [32*v + 8c, 32*v + 8c + 8) for v < KV.  Rows past
    // the end (scores the caller drops) load the last row instead: the loads stay unconditional,
    // so none waits at a branch join before the next is issued.
    const int64_t rl = min(r0 + g, nrows - 1), rh = min(r0 + g + 8, nrows - 1);
#pragma unroll
    for (int v = 0; v < KV; ++v) {
        lo[v] = ld_stream(keys + rl * (KV * 32) + v * 32 + c * 8, pol);
        hi[v] = ld_stream(keys + rh * (KV * 32) + v * 32 + c * 8, pol);
    }
}

template <int KV>
__device__ __forceinline__ void score16(const uint4 (&lo)[KV], const uint4 (&hi)[KV], const uint32_t (&bq)[2 * KV][2],
                                        const float (&wv)[2], float& s_lo, float& s_hi) {
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

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Streaming 8-byte load (see ld_stream).
__device__ __forceinline__ uint2 ld_stream8(const void* p, uint64_t pol) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0,%1}, [%2], %3;"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p), "l"(pol));
    return v;
}

// x * 2^e, correctly rounded (the same value as ldexpf): a multiply by the power of two built from
// its exponent bits when 2^e is a normal float, else ldexpf itself.
__device__ __forceinline__ float scale_pow2(float x, int e) {
    return (e >= -126 && e <= 127) ? __fmul_rn(x, __uint_as_float((uint32_t)(e + 127) << 23)) : ldexpf(x, e);
}

// Two E4M3 values (low byte first) to two f16 values (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "h"((unsigned short)two_bytes));
    return r;
}

// Scores of 16 consecutive entries with 8-bit block-scaled keys (blocks of 32 channels, E4M3
// elements, one power-of-two scale byte per block): thread (g, c) loads 8 bytes of each block for
// rows g and g + 8 (load16_mx8), converts them to f16 (exact), and the products with the f16 query
// (each head pre-scaled by a power of two 2^qsh[.], so it is exact in f16) accumulate per block in
// fp32; the block scales and the query scale are applied exactly (powers of two) before relu
// (score16_mx8).
template <int NB>
struct Keys8 {
    uint2 lo[NB], hi[NB];
    uint32_t sl, sh;  // scale bytes of rows g and g + 8
};

template <int NB>
__device__ __forceinline__ void load16_mx8(const uint8_t* keys, const uint8_t* scales, int64_t r0, int64_t nrows,
                                           int g, int c, uint64_t pol, Keys8<NB>& k) {
    constexpr int DI = 32 * NB;
    // rows past the end (scores the caller drops) load the last row: unconditional loads (see load16)
    const int64_t rl = min(r0 + g, nrows - 1), rh = min(r0 + g + 8, nrows - 1);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        k.lo[b] = ld_stream8(keys + rl * DI + b * 32 + c * 8, pol);
        k.hi[b] = ld_stream8(keys + rh * DI + b * 32 + c * 8, pol);
    }
    k.sl = NB == 2 ? (uint32_t)*reinterpret_cast<const uint16_t*>(scales + rl * NB) : scales[rl];
    k.sh = NB == 2 ? (uint32_t)*reinterpret_cast<const uint16_t*>(scales + rh * NB) : scales[rh];
}

template <int NB>
__device__ __forceinline__ void score16_mx8(const Keys8<NB>& k, const uint32_t (&bq)[2 * NB][2], const float (&wv)[2],
                                            const int (&qsh)[2], float& s_lo, float& s_hi) {
    float tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const uint32_t l0 = e4m3x2_to_f16x2(k.lo[b].x), l1 = e4m3x2_to_f16x2(k.lo[b].x >> 16);
        const uint32_t l2 = e4m3x2_to_f16x2(k.lo[b].y), l3 = e4m3x2_to_f16x2(k.lo[b].y >> 16);
        const uint32_t h0 = e4m3x2_to_f16x2(k.hi[b].x), h1 = e4m3x2_to_f16x2(k.hi[b].x >> 16);
        const uint32_t h2 = e4m3x2_to_f16x2(k.hi[b].y), h3 = e4m3x2_to_f16x2(k.hi[b].y >> 16);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t a0[4] = {l0, h0, l1, h1};
        const uint32_t a1[4] = {l2, h2, l3, h3};
        mma_f16_16816(acc, a0, bq[2 * b]);
        mma_f16_16816(acc, a1, bq[2 * b + 1]);
        const int el = (int)((k.sl >> (8 * b)) & 0xFFu) - 127, eh = (int)((k.sh >> (8 * b)) & 0xFFu) - 127;
        tot[0] = __fadd_rn(tot[0], scale_pow2(acc[0], el - qsh[0]));
        tot[1] = __fadd_rn(tot[1], scale_pow2(acc[1], el - qsh[1]));
        tot[2] = __fadd_rn(tot[2], scale_pow2(acc[2], eh - qsh[0]));
        tot[3] = __fadd_rn(tot[3], scale_pow2(acc[3], eh - qsh[1]));
    }
    float pl = wv[0] * fmaxf(tot[0], 0.f) + wv[1] * fmaxf(tot[1], 0.f);
    float ph = wv[0] * fmaxf(tot[2], 0.f) + wv[1] * fmaxf(tot[3], 0.f);
    pl += __shfl_xor_sync(0xffffffffu, pl, 1);
    ph += __shfl_xor_sync(0xffffffffu, ph, 1);
    pl += __shfl_xor_sync(0xffffffffu, pl, 2);
    ph += __shfl_xor_sync(0xffffffffu, ph, 2);
    s_lo = pl;
    s_hi = ph;
}

// ---- block-wide helpers ---------------------------------------------------------------------

// Bring `bytes` (a multiple of 16, 16-byte aligned) at `src` into L2 without waiting for them.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t composite(uint32_t key, int64_t j) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

// Query qi's indices are out: publish its ready word (one thread, after the stores it covers are
// ordered before it: by a CTA barrier, or by the grid dependency for the scan's own results).
__device__ __forceinline__ void signal_ready(const IndexParams& p, int qi) {
    if (!p.ready || p.debug_fault == 2) return;  // fault injection: the waits on the word run out
    __threadfence();
    st_release_gpu(p.ready + qi, 1u);
}


// Exclusive prefix of one value per thread; *total gets the block's sum.  wsum: NT/32 words.
// Two barriers: the warps' totals are published, then every warp sums the ones before it.
template <int NT>
__device__ __forceinline__ uint32_t excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const uint32_t x = wsum[w];
        before += w < warp ? x : 0u;
        all += x;
    }
    *total = all;
    __syncthreads();  // wsum may be written again after the return
    return before + incl - v;
}

// Over BINS bins: the unique bin b with suffix(b) >= target > suffix(b + 1), where suffix(b) =
// sum of hist[b' >= b] (target >= 1).  out[0] = b (0xFFFFFFFF if the total is below target),
// out[1] = suffix(b + 1), out[2] = suffix(b).  Thread t owns BINS/NT consecutive bins counted
// from the top, so a forward scan over threads is a suffix scan over bins; it reads them with
// 16-byte loads (hist 16-byte aligned; a quarter-warp's loads cover all banks once).
template <int NT, int BINS = kHistBins>
__device__ void find_bin(const uint32_t* hist, uint32_t target, uint32_t* wsum, uint32_t* out) {
    constexpr int PER = BINS / NT;
    static_assert(PER % 4 == 0, "find_bin reads its bins as 16-byte vectors");
    const int t = threadIdx.x;
    const int b0 = PER * (NT - 1 - t);  // bins [b0, b0 + PER)
    uint32_t h[PER];
#pragma unroll
    for (int i = 0; i < PER / 4; ++i) {
        const uint4 v = reinterpret_cast<const uint4*>(hist + b0)[i];
        h[4 * i] = v.x; h[4 * i + 1] = v.y; h[4 * i + 2] = v.z; h[4 * i + 3] = v.w;
    }
    uint32_t part = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) part += h[i];
    if (t == 0) out[0] = 0xFFFFFFFFu;
    uint32_t total;
    uint32_t above = excl_scan<NT>(part, wsum, &total);  // bins above b0 + PER - 1
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
        const uint32_t here = above + h[i];
        if (here >= target && above < target) { out[0] = (uint32_t)(b0 + i); out[1] = above; out[2] = here; }
        above = here;
    }
    __syncthreads();
}

// A list of 64-bit keys, in shared or global memory.
struct KeyList {
    const uint64_t* smem;
    const uint64_t* gmem;
    __device__ __forceinline__ uint64_t get(uint32_t i) const {
        return smem ? smem[i] : __ldcg(reinterpret_cast<const unsigned long long*>(gmem) + i);
    }
};

// The key T with exactly `need` of the list's members of bin `top` (their top BITS bits) at or above
// it: radix passes of BITS bits below the top BITS, counted with shared-memory atomics in
// cnt[1 << BITS]; stops as soon as the chosen digit holds exactly the remaining count.
template <int NT, int BITS>
__device__ uint64_t radix_select(const KeyList& L, uint32_t n, uint32_t need, uint32_t top, uint32_t* cnt,
                                 uint32_t* wsum, uint32_t* res) {
    constexpr int kBins = 1 << BITS;
    uint64_t prefix = (uint64_t)top << (64 - BITS);
    uint64_t mask = (uint64_t)(kBins - 1) << (64 - BITS);
    uint32_t remaining = need;
    for (int shift = 64 - 2 * BITS;; shift -= BITS) {
        const int sh = shift < 0 ? 0 : shift;
        const int bits = shift < 0 ? BITS + shift : BITS;
        const uint32_t dmask = (1u << bits) - 1u;
        for (int i = threadIdx.x; i < kBins; i += NT) cnt[i] = 0;
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < n; i += NT) {
            const uint64_t v = L.get(i);
            if ((v & mask) == prefix) atomicAdd(&cnt[(uint32_t)(v >> sh) & dmask], 1u);
        }
        __syncthreads();
        find_bin<NT, kBins>(cnt, remaining, wsum, res);
        const uint32_t dg = res[0], above = res[1], in_digit = res[2] - res[1];
        __syncthreads();
        remaining -= above;
        prefix |= (uint64_t)dg << sh;
        mask |= (uint64_t)dmask << sh;
        if (in_digit == remaining || sh == 0) return prefix;  // lower bits left at zero
    }
}

// Ordered compaction of one round of NT * PER items laid out warp-contiguously: lane l of warp w
// holds item w * 32 * PER + u * 32 + l of the round as v[u], a member when keep[u].  Every load
// of such a layout reads 32 consecutive items; the members keep item order through one ballot per
// u and one block scan over the warps' counts.  write(written + rank, v) is called for each member
// (rank = its place among the round's members); returns the round's member count (every thread).
template <int NT, int PER, typename Write>
__device__ __forceinline__ uint32_t compact_round(const uint64_t (&v)[PER], const bool (&keep)[PER], uint32_t written,
                                                  Write&& write, uint32_t* wsum) {
    const int lane = threadIdx.x & 31;
    uint32_t mask[PER];
    uint32_t cnt = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        mask[u] = __ballot_sync(0xffffffffu, keep[u]);
        cnt += __popc(mask[u]);
    }
    uint32_t tot;
    const uint32_t ex = excl_scan<NT>(lane == 0 ? cnt : 0u, wsum, &tot);
    uint32_t off = written + __shfl_sync(0xffffffffu, ex, 0);
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        if (keep[u]) write(off + __popc(mask[u] & lt), v[u]);
        off += __popc(mask[u]);
    }
    return tot;
}

// Distributed shared memory: store 8 bytes / a word at the location `p` (an address in this CTA's
// shared memory) in the CTA of rank `rank`, and load a word from there.
__device__ __forceinline__ void st_cluster_u64(const void* p, uint32_t rank, uint64_t v) {
    uint32_t a;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(a), "l"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(const void* p, uint32_t rank, uint32_t v) {
    uint32_t a;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_cluster_u32(const void* p, uint32_t rank) {
    uint32_t a, v;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}

constexpr int kListKeys = 4096;                  // keys of the final list held in shared memory
constexpr int kTailPer = 8;                      // items per thread and round of an ordered compaction
constexpr int kScanDynSmem = kListKeys * 8;      // dynamic shared memory: chunk scores, then the list
constexpr int64_t kScanChunkMax = kScanDynSmem / 4;
static_assert(kScanChunkMax >= 512, "a chunk holds at least one pass of the scan");

// Scores of the selected entries of a query that selects all of its E <= k entries (recomputed; E is
// small), written to sout[0..E).
__device__ void scores_of_all(const IndexParams& p, int qi, int64_t csa_off, int64_t E, float* sout) {
    for (int64_t j = threadIdx.x; j < E; j += blockDim.x) {
        float s = 0.f;
        for (int h = 0; h < p.H_I; ++h) {
            const uint16_t* qh = p.q_idx + ((int64_t)qi * p.H_I + h) * p.d_I;
            float dot = 0.f;
            for (int cc = 0; cc < p.d_I; ++cc) {
                float k;
                if (p.keys_q) {  // the dequantized 8-bit key: 2^e times the E4M3 value
                    const uint32_t two = e4m3x2_to_f16x2(p.keys_q[(csa_off + j) * p.d_I + cc]);
                    const int e = (int)p.key_scales[(csa_off + j) * (p.d_I / 32) + cc / 32] - 127;
                    k = ldexpf(__low2float(*reinterpret_cast<const __half2*>(&two)), e);
                } else {
                    k = __uint_as_float((uint32_t)p.entry_keys[(csa_off + j) * p.d_I + cc] << 16);
                }
                dot = fmaf(__uint_as_float((uint32_t)qh[cc] << 16), k, dot);
            }
            s += p.w[(int64_t)qi * p.H_I + h] * fmaxf(dot, 0.f);
        }
        sout[j] = s;
    }
}

// 8-bit block-scaled copies of stored bf16 indexer keys: 8 threads per entry (4 per 32-channel block),
// entries [r0, r1) of sequence b (ranges as csa_compress).
__global__ void __launch_bounds__(256) quantize_keys_kernel(const csa_seq* seqs, const int64_t* ranges, int m, int d_I,
                                                            const uint16_t* keys, uint8_t* keys_q, uint8_t* scales,
                                                            int* status) {
    const int b = blockIdx.y;
    const int tpe = d_I / 8;  // threads per entry: 8 or 4
    const int64_t e0 = ranges[2 * b], e1 = ranges[2 * b + 1];
    const csa_seq sq = seqs[b];
    if (e0 < 0 || e1 < e0 || (int64_t)m * e1 > sq.len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(status, CSA_ERR_INDEX);
        return;
    }
    const int lane = threadIdx.x & 31, sub = threadIdx.x / tpe, g = threadIdx.x % tpe;
    const unsigned mask = 0xFu << (lane & ~3);
    for (int64_t j = e0 + (int64_t)blockIdx.x * (256 / tpe) + sub; j < e1; j += (int64_t)gridDim.x * (256 / tpe)) {
        const int64_t row = sq.csa_off + j;
        const uint4 kb = *reinterpret_cast<const uint4*>(keys + row * d_I + 8 * g);
        uint32_t sb;
        const uint2 q = quant_mx8(kb, mask, &sb);
        *reinterpret_cast<uint2*>(keys_q + row * d_I + 8 * g) = q;
        if ((g & 3) == 0) scales[row * (d_I / 32) + g / 4] = (uint8_t)sb;
    }
}

// ---- prefill select ---------------------------------------------------------------------------
//
// One CTA per query over a stored score row of at most kSelBufMax entries: the row is staged in
// shared memory by bulk copies; a histogram of a strided sample of 4,096 scores gives a bin above
// which about 2k/n of the sample lies, low enough that at least k entries pass it with overwhelming
// probability; every entry of that bin and above is kept, in index order (the whole row instead if
// fewer than k passed); the candidates' own histogram gives the exact threshold bin, a radix select
// inside it the threshold, and the k indices are compacted in ascending order.

constexpr int kSelPerMax = 64;                           // scores per thread
constexpr int kSelBufMax = kSelPerMax * kSelectThreads;  // scores of one row (shared memory)
constexpr int kSelListMax = 8192;                        // kept keys held in shared memory

struct SelSmem {
    static constexpr int kHist = 0;                         // u32[kHistBins]
    static constexpr int kList = kHist + kHistBins * 4;     // u64[kSelListMax]
    static constexpr int kBuf = kList + kSelListMax * 8;    // f32[buf]
    static constexpr size_t bytes(int64_t buf) { return (size_t)kBuf + (size_t)buf * 4; }
};

__global__ void __launch_bounds__(kSelectThreads) index_select_kernel(IndexParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw + SelSmem::kHist);
    uint64_t* slist = reinterpret_cast<uint64_t*>(smem_raw + SelSmem::kList);
    float* sbuf = reinterpret_cast<float*>(smem_raw + SelSmem::kBuf);
    __shared__ uint32_t s_wsum[kSelectThreads / 32];
    __shared__ uint32_t s_res[4];
    __shared__ uint64_t s_bar;
    grid_dep_wait();  // the scores come from the prefill GEMM
    grid_dep_launch();
    const int qi = blockIdx.x, tid = threadIdx.x;
    const csa_query qr = p.queries[qi];
    const bool seq_ok = qr.seq >= 0 && qr.reserved == 0;
    const csa_seq sq = seq_ok ? p.seqs[qr.seq] : csa_seq{0, 0, 0, 0};
    const bool valid = seq_ok && qr.len >= 1 && qr.len <= sq.len;
    const int64_t E = valid ? qr.len / p.m : 0;
    int32_t* out = p.idx_out + (int64_t)qi * p.k;
    float* sout = p.score_out ? p.score_out + (int64_t)qi * p.k : nullptr;
    if (!valid || E > p.max_entries || E > kSelBufMax || E <= p.k) {
        const bool bad = !valid || E > p.max_entries || E > kSelBufMax;
        if (bad && tid == 0) report(p.status, CSA_ERR_INDEX);
        const int64_t n = bad ? 0 : E;
        for (int i = tid; i < p.k; i += kSelectThreads) {
            out[i] = i < n ? i : -1;
            if (sout) sout[i] = __int_as_float(0x7FC00000);
        }
        if (sout && n > 0) {
            __syncthreads();
            scores_of_all(p, qi, sq.csa_off, n, sout);
        }
        return;
    }
    const int n = (int)E;
    const float* srow = p.scores + (int64_t)qi * p.e_stride;
    // 1. the row into shared memory (bulk copies of the 16-byte-multiple part, then the tail)
    const int n16 = n & ~3;
    if (tid == 0) {
        mbar_init(&s_bar, 1);
        fence_mbar_init();
        const uint32_t bytes = (uint32_t)n16 * 4u;
        mbar_arrive_expect_tx(&s_bar, bytes);
        for (uint32_t off = 0; off < bytes; off += 65536u)
            bulk_load(smem_u32(sbuf) + off, srow + off / 4u, min(65536u, bytes - off), &s_bar);
    }
    if (tid < n - n16) sbuf[n16 + tid] = __ldg(srow + n16 + tid);
    __syncthreads();
    if (!__syncthreads_and(mbar_wait(&s_bar, 0, p.status, nullptr) ? 1 : 0)) return;  // timeout recorded
    // 2. threshold bin estimated from a sample
    for (int i = tid; i < kHistBins; i += kSelectThreads) hist[i] = 0u;
    __syncthreads();
    const int S = n < 4096 ? n : 4096;
    for (int i = tid; i < S; i += kSelectThreads) atomicAdd(&hist[float_key(sbuf[((int64_t)i * n) / S]) >> 21], 1u);
    __syncthreads();
    const int64_t want = (2 * (int64_t)p.k * S + n - 1) / n;
    find_bin<kSelectThreads>(hist, (uint32_t)(want < S ? want : S + 1), s_wsum, s_res);
    uint32_t b_lo = s_res[0] == 0xFFFFFFFFu ? 0u : s_res[0];  // no bin qualifies: keep everything
    // 3. candidates: the entries of bin >= b_lo in index order, in shared memory or (a long list) in
    //    the query's global segment
    const int L = (n + kSelectThreads - 1) / kSelectThreads;  // entries per thread
    const int i0 = tid * L, i1 = min(n, i0 + L);
    uint64_t* gseg = p.seg + (int64_t)qi * p.e_seg;
    uint32_t n_cand = 0;
    bool in_smem = true;
    for (int pass = 0; pass < 2; ++pass) {
        uint32_t mine = 0;
        for (int i = i0; i < i1; ++i) mine += (float_key(sbuf[i]) >> 21) >= b_lo ? 1u : 0u;
        uint32_t tot;
        uint32_t o = excl_scan<kSelectThreads>(mine, s_wsum, &tot);
        if (tot < (uint32_t)p.k && b_lo > 0) {  // the estimate was too high (rare): keep everything
            b_lo = 0;
            continue;
        }
        in_smem = tot <= (uint32_t)kSelListMax;
        uint64_t* dst = in_smem ? slist : gseg;
        for (int i = i0; i < i1; ++i) {
            const uint32_t key = float_key(sbuf[i]);
            if ((key >> 21) >= b_lo) dst[o++] = composite(key, i);
        }
        n_cand = tot;
        break;
    }
    __syncthreads();
    // 4. the exact threshold bin from the candidates' own histogram, then the radix select
    const KeyList KL{in_smem ? slist : nullptr, in_smem ? nullptr : gseg};
    for (int i = tid; i < kHistBins; i += kSelectThreads) hist[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < n_cand; i += kSelectThreads) atomicAdd(&hist[(uint32_t)(KL.get(i) >> 53)], 1u);
    __syncthreads();
    find_bin<kSelectThreads>(hist, (uint32_t)p.k, s_wsum, s_res);
    const uint32_t b1 = s_res[0], above = s_res[1], n_bin = s_res[2] - s_res[1];
    if (b1 == 0xFFFFFFFFu) {  // fewer than k candidates: cannot happen (the whole row was kept)
        if (tid == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const uint32_t need = (uint32_t)p.k - above;
    const uint64_t T = need == n_bin ? ((uint64_t)b1 << 53)
                                     : radix_select<kSelectThreads, 11>(KL, n_cand, need, b1, hist, s_wsum, s_res);
    // 5. compaction in index order
    const uint32_t per_t = (n_cand + kSelectThreads - 1) / kSelectThreads;
    const uint32_t j0 = tid * per_t, j1 = min(n_cand, j0 + per_t);
    uint32_t mine = 0;
    for (uint32_t i = j0; i < j1; ++i) mine += KL.get(i) >= T ? 1u : 0u;
    uint32_t kept_total;
    uint32_t o = excl_scan<kSelectThreads>(mine, s_wsum, &kept_total);
    for (uint32_t i = j0; i < j1; ++i) {
        const uint64_t v = KL.get(i);
        if (v >= T) {
            if (o < (uint32_t)p.k) {
                out[o] = (int32_t)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
                if (sout) sout[o] = key_float((uint32_t)(v >> 32));
            }
            ++o;
        }
    }
    if (tid == 0 && kept_total != (uint32_t)p.k) report(p.status, CSA_ERR_INDEX);
}

// ---- exact top-k inside the scan grid -------------------------------------------------------------
//
// When every scan CTA is resident at once (the grid fits the SMs), the CTAs of query qi finish the
// selection themselves, meeting on the query's counters qs[0..2]:
//   A. each CTA adds its histogram to the query's and counts itself in qs[0]; once all nch chunks
//      have, every CTA reads the complete histogram and finds the threshold bin b1;
//   B. each CTA counts its members (its scores of bin >= b1, still in shared memory), publishes the
//      count and counts itself in qs[1]; once all counts are out, it stores its members in index
//      order at its place (the counts of the chunks before it) of the query's list;
//   C. the last CTA to count itself in qs[2] radix-selects the exact threshold inside bin b1 among
//      the list's members, writes the k indices in ascending order and publishes the ready word.
// Every wait is bounded (a wait that runs out records CSA_ERR_TIMEOUT; the CTA gives up).
__device__ void scan_select(const IndexParams& p, int qi, int cidx, int nch, int64_t c0, int n, const float* ssc,
                            uint64_t* slist, uint32_t* hist, uint32_t* s_wsum, uint32_t* s_res, int32_t* out,
                            float* sout, int64_t csa_off) {
    __shared__ int s_ok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t* qs = p.qsync + (int64_t)qi * 4;
    // A. the query's complete histogram and its threshold bin
    __syncthreads();  // this CTA's histogram atomics are issued
    if (tid == 0) {
        __threadfence();
        atomicAdd(qs + 0, 1u);
        s_ok = count_wait(qs + 0, (uint32_t)nch, p.status, nullptr) ? 1 : 0;
    }
    __syncthreads();
    if (!s_ok) return;
    {
        const uint32_t* gh = p.hist + (int64_t)qi * kKeyBins;
        uint32_t hv[kKeyBins / kScanThreads];
#pragma unroll
        for (int i = 0; i < kKeyBins / kScanThreads; ++i) hv[i] = __ldcg(gh + tid + i * kScanThreads);
#pragma unroll
        for (int i = 0; i < kKeyBins / kScanThreads; ++i) hist[tid + i * kScanThreads] = hv[i];
    }
    __syncthreads();
    find_bin<kScanThreads, kKeyBins>(hist, (uint32_t)p.k, s_wsum, s_res);
    const uint32_t b1 = s_res[0], above = s_res[1], at = s_res[2];
    const bool bad = b1 == 0xFFFFFFFFu;  // fewer than k scores: cannot happen for E > k
    // B. this chunk's members: count, publish, wait for every chunk's count, then store them
    uint32_t mine = 0;
    for (int i = tid; i < n; i += kScanThreads) mine += (!bad && (float_key(ssc[i]) >> (32 - kKeyBits)) >= b1) ? 1u : 0u;
    uint32_t cnt;
    (void)excl_scan<kScanThreads>(mine, s_wsum, &cnt);
    uint32_t* counts = p.meta + (int64_t)qi * p.max_chunks;
    if (tid == 0) {
        counts[cidx] = cnt;
        __threadfence();
        atomicAdd(qs + 1, 1u);
        s_ok = count_wait(qs + 1, (uint32_t)nch, p.status, nullptr) ? 1 : 0;
    }
    __syncthreads();
    if (!s_ok) return;
    uint32_t before = 0;
    for (int j = tid; j < cidx; j += kScanThreads) before += __ldcg(counts + j);
    uint32_t off;
    (void)excl_scan<kScanThreads>(before, s_wsum, &off);
    uint64_t* lst = p.seg + (int64_t)qi * p.e_seg;
    {
        uint32_t written = 0;
        for (int base = 0; base < n; base += kScanThreads * kTailPer) {
            const int first = base + warp * 32 * kTailPer + lane;
            uint64_t v[kTailPer];
            bool keep[kTailPer];
#pragma unroll
            for (int u = 0; u < kTailPer; ++u) {
                const int i = first + u * 32;
                const uint32_t key = i < n ? float_key(ssc[i]) : 0u;
                keep[u] = !bad && i < n && (key >> (32 - kKeyBits)) >= b1;
                v[u] = composite(key, c0 + i);
            }
            written += compact_round<kScanThreads, kTailPer>(
                v, keep, written, [&](uint32_t pos, uint64_t x) { lst[off + pos] = x; }, s_wsum);
        }
    }
    // C. the last chunk of the query selects
    __syncthreads();  // every member store of the CTA precedes the count
    if (tid == 0) {
        __threadfence();
        s_ok = atomicAdd(qs + 2, 1u) == (uint32_t)nch - 1 ? 1 : 0;
    }
    __syncthreads();
    if (!s_ok) return;
    __threadfence();  // the other chunks' members, stored before their counts, are visible
    if (bad) {
        if (tid == 0) {
            report(p.status, CSA_ERR_INDEX);
            signal_ready(p, qi);
        }
        return;
    }
    const uint32_t n_tot = at, need = (uint32_t)p.k - above, n_bin = at - above;
    const bool in_smem = n_tot <= (uint32_t)kListKeys;
    if (in_smem) {
        for (uint32_t i = tid; i < n_tot; i += kScanThreads) slist[i] = __ldcg(reinterpret_cast<const unsigned long long*>(lst) + i);
        __syncthreads();
    }
    const KeyList L{in_smem ? slist : nullptr, in_smem ? nullptr : lst};
    const uint64_t T = need == n_bin ? ((uint64_t)b1 << (64 - kKeyBits))
                                     : radix_select<kScanThreads, kKeyBits>(L, n_tot, need, b1, hist, s_wsum, s_res);
    uint32_t kept = 0;
    for (uint32_t base = 0; base < n_tot; base += kScanThreads * kTailPer) {
        const uint32_t first = base + (uint32_t)(warp * 32 * kTailPer + lane);
        uint64_t v[kTailPer];
        bool keep[kTailPer];
#pragma unroll
        for (int u = 0; u < kTailPer; ++u) {
            const uint32_t i = first + u * 32;
            v[u] = i < n_tot ? L.get(i) : 0ull;
            keep[u] = i < n_tot && v[u] >= T;
        }
        kept += compact_round<kScanThreads, kTailPer>(v, keep, kept, [&](uint32_t o, uint64_t x) {
            if (o < (uint32_t)p.k) {
                out[o] = (int32_t)(0xFFFFFFFFu - (uint32_t)(x & 0xFFFFFFFFull));
                if (sout) sout[o] = key_float((uint32_t)(x >> 32));
            }
        }, s_wsum);
    }
    if (tid == 0 && kept != (uint32_t)p.k) report(p.status, CSA_ERR_INDEX);
    __syncthreads();  // every index store of the CTA precedes the release
    if (tid == 0) signal_ready(p, qi);
    // the attention that follows gathers the selected rows: start bringing them into L2
    if (p.prefetch_rows)
        for (int o = tid; o < p.k; o += kScanThreads) {
            const int32_t j = __ldcg(out + o);
            if (j >= 0) prefetch_l2(p.prefetch_rows + (csa_off + j) * p.prefetch_row_bytes, p.prefetch_row_bytes);
        }
}

// ---- decode scan ------------------------------------------------------------------------------------
//
// Scan CTA (chunk c, query qi): the scores of entries [c*chunk, min(E, (c+1)*chunk)) on the tensor
// cores, written to the score row and kept in shared memory, counted into the query's histogram of
// the top kKeyBits bits of the order-preserving score key; then the chunk's candidates -- its
// entries of bin >= b_c, b_c the highest bin that still leaves at least kloc entries (kloc about
// twice the chunk's expected share of the top-k) -- go to the candidate buffer in index order, with
// b_c.
// index_final_kernel selects the exact top-k from them.
template <int KV, bool MX8>
__global__ void __launch_bounds__(kScanThreads, 2) index_scan_kernel(IndexParams p) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ __align__(16) uint32_t hist[kKeyBins];
    __shared__ float sc[kScanThreads / 32][4][16];
    __shared__ uint32_t s_wsum[kScanThreads / 32];
    __shared__ uint32_t s_res[4];
    float* ssc = reinterpret_cast<float*>(dsm);  // the chunk's scores
    grid_dep_wait();  // the query table may come from the previous kernel
    grid_dep_launch();
    const int qi = blockIdx.y;
    const int tid = threadIdx.x;
    const csa_query qr = p.queries[qi];
    const bool seq_ok = qr.seq >= 0 && qr.reserved == 0;
    const csa_seq sq = seq_ok ? p.seqs[qr.seq] : csa_seq{0, 0, 0, 0};
    const bool valid = seq_ok && qr.len >= 1 && qr.len <= sq.len;
    const int64_t E = valid ? qr.len / p.m : 0;
    int32_t* out = p.idx_out + (int64_t)qi * p.k;
    float* sout = p.score_out ? p.score_out + (int64_t)qi * p.k : nullptr;
    if (!valid || E > p.max_entries || E <= p.k) {
        // an invalid query (reported, nothing selected) or one that selects everything: chunk 0 alone
        if (blockIdx.x != 0) return;
        const bool bad = !valid || E > p.max_entries;
        if (bad && tid == 0) report(p.status, CSA_ERR_INDEX);
        const int64_t n = bad ? 0 : E;
        for (int i = tid; i < p.k; i += kScanThreads) {
            out[i] = i < n ? i : -1;
            if (sout) sout[i] = __int_as_float(0x7FC00000);
        }
        if (sout && n > 0) {
            __syncthreads();
            scores_of_all(p, qi, sq.csa_off, n, sout);
        }
        if (p.qsync) {  // no final select follows: publish the ready word here
            __syncthreads();
            if (tid == 0) signal_ready(p, qi);
        }
        return;
    }
    const int64_t chunk = p.chunk;
    const int nch = (int)((E + chunk - 1) / chunk);
    const int cidx = blockIdx.x;
    if (cidx >= nch) return;
    const int64_t c0 = (int64_t)cidx * chunk;
    const int64_t c1 = min(E, c0 + chunk);
    for (int i = tid; i < kKeyBins; i += kScanThreads) hist[i] = 0u;

    const int lane = tid & 31, warp = tid >> 5;
    {
        const int g = lane >> 2, c = lane & 3;
        // B fragments (query, permuted exactly like the key loads) and head weights
        uint32_t bq[2 * KV][2];
        float wv[2];
        int qsh[2] = {0, 0};  // 8-bit keys: the power-of-two pre-scale of heads 2c and 2c + 1
        const uint16_t* qrow = p.q_idx + ((int64_t)qi * p.H_I + g) * p.d_I;
        const bool hv = g < p.H_I;
        uint4 qv[KV];
#pragma unroll
        for (int v = 0; v < KV; ++v)
            qv[v] = hv ? *reinterpret_cast<const uint4*>(qrow + v * 32 + c * 8) : make_uint4(0, 0, 0, 0);
        if (!MX8) {
#pragma unroll
            for (int v = 0; v < KV; ++v) {
                bq[2 * v][0] = qv[v].x; bq[2 * v][1] = qv[v].y;
                bq[2 * v + 1][0] = qv[v].z; bq[2 * v + 1][1] = qv[v].w;
            }
        } else {
            // head g's query in f16, scaled by 2^s with s chosen so that its largest magnitude lies in
            // [2^14, 2^15): exact in f16 (down to 2^-31 of that magnitude) and far from overflow
            float f[KV][8];
            float amax = 0.f;
#pragma unroll
            for (int v = 0; v < KV; ++v) {
                unpack8(qv[v], f[v]);
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[v][i]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            int ex = 0;
            if (amax > 0.f) frexpf(amax, &ex);  // amax in [2^(ex-1), 2^ex)
            const int sg = amax > 0.f ? 15 - ex : 0;
#pragma unroll
            for (int v = 0; v < KV; ++v) {
                uint32_t h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 t = __floats2half2_rn(ldexpf(f[v][2 * i], sg), ldexpf(f[v][2 * i + 1], sg));
                    h[i] = *reinterpret_cast<const uint32_t*>(&t);
                }
                bq[2 * v][0] = h[0]; bq[2 * v][1] = h[1];
                bq[2 * v + 1][0] = h[2]; bq[2 * v + 1][1] = h[3];
            }
            // heads 2c and 2c + 1 live in the quads of rows 2c and 2c + 1
            qsh[0] = __shfl_sync(0xffffffffu, sg, (2 * c) * 4);
            qsh[1] = __shfl_sync(0xffffffffu, sg, (2 * c + 1) * 4);
        }
        const int h0 = 2 * c, h1 = 2 * c + 1;
        wv[0] = h0 < p.H_I ? p.w[(int64_t)qi * p.H_I + h0] : 0.f;
        wv[1] = h1 < p.H_I ? p.w[(int64_t)qi * p.H_I + h1] : 0.f;
        __syncthreads();

        const uint16_t* keys = p.entry_keys + sq.csa_off * p.d_I;
        float* srow = p.scores + (int64_t)qi * p.e_stride;
        const uint64_t pol = policy_evict_first();
        // a pass's scores: staged in shared memory, then stored coalesced and counted (groups u of
        // 16 rows at base + (u * 8 + warp) * 16)
        auto finish = [&](int64_t base, const float (&s)[4][2], int groups) {
            if (c == 0) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (u < groups) { sc[warp][u][g] = s[u][0]; sc[warp][u][g + 8] = s[u][1]; }
            }
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (u < groups && lane < 16) {
                    const int64_t r = base + (int64_t)(u * (kScanThreads / 32) + warp) * 16 + lane;
                    if (r < c1) {
                        const float v = sc[warp][u][lane];
                        srow[r] = v;
                        ssc[r - c0] = v;
                        atomicAdd(&hist[float_key(v) >> (32 - kKeyBits)], 1u);
                    }
                }
            }
            __syncwarp();
        };
        if (MX8) {
            constexpr int kRowsPerPass = kScanThreads / 32 * 16 * 4;  // 512 entries: 4 groups of 16 per warp
            for (int64_t base = c0; base < c1; base += kRowsPerPass) {
                float s[4][2];
                // every load of the pass first, then the scores
                Keys8<KV> k8[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    load16_mx8<KV>(p.keys_q + sq.csa_off * p.d_I, p.key_scales + sq.csa_off * KV,
                                   base + (int64_t)(u * (kScanThreads / 32) + warp) * 16, c1, g, c, pol, k8[u]);
#pragma unroll
                for (int u = 0; u < 4; ++u) score16_mx8<KV>(k8[u], bq, wv, qsh, s[u][0], s[u][1]);
                finish(base, s, 4);
            }
        } else {
            // software pipeline over passes of two 16-row groups per warp, in two register buffers:
            // the next pass's loads are in flight while this pass is scored (a warp never waits with
            // no loads outstanding).  Loads past the chunk read its last row; their scores are dropped.
            constexpr int kG = 2;
            constexpr int64_t kRows = kScanThreads / 32 * 16 * kG;  // 256 entries per pass
            uint4 alo[kG][KV], ahi[kG][KV], blo[kG][KV], bhi[kG][KV];
            auto load_pass = [&](int64_t base, uint4 (&lo)[kG][KV], uint4 (&hi)[kG][KV]) {
#pragma unroll
                for (int u = 0; u < kG; ++u)
                    load16<KV>(keys, base + (int64_t)(u * (kScanThreads / 32) + warp) * 16, c1, g, c, pol, lo[u], hi[u]);
            };
            auto score_pass = [&](int64_t base, const uint4 (&lo)[kG][KV], const uint4 (&hi)[kG][KV]) {
                float s[4][2];
#pragma unroll
                for (int u = 0; u < kG; ++u) score16<KV>(lo[u], hi[u], bq, wv, s[u][0], s[u][1]);
                finish(base, s, kG);
            };
            load_pass(c0, alo, ahi);
            for (int64_t base = c0; base < c1; base += 2 * kRows) {
                load_pass(base + kRows, blo, bhi);
                score_pass(base, alo, ahi);
                load_pass(base + 2 * kRows, alo, ahi);
                score_pass(base + kRows, blo, bhi);
            }
        }
    }
    __syncthreads();
    {
        uint32_t* gh = p.hist + (int64_t)qi * kKeyBins;
        for (int i = tid; i < kKeyBins; i += kScanThreads)
            if (hist[i]) atomicAdd(&gh[i], hist[i]);
    }
    if (p.qsync) {  // the scan grid selects (see scan_select)
        scan_select(p, qi, cidx, nch, c0, (int)(c1 - c0), ssc, reinterpret_cast<uint64_t*>(dsm), hist, s_wsum, s_res,
                    out, sout, sq.csa_off);
        return;
    }
    // ---- the chunk's candidates
    const int n = (int)(c1 - c0);
    const int cap = p.cand_cap;
    const int64_t kloc64 = (2 * (int64_t)p.k * n + E - 1) / E + 16;
    const uint32_t kloc = (uint32_t)min((int64_t)cap, min((int64_t)n, kloc64));
    find_bin<kScanThreads, kKeyBins>(hist, kloc, s_wsum, s_res);
    uint32_t bc = s_res[0] == 0xFFFFFFFFu ? 0u : s_res[0];
    if (s_res[0] != 0xFFFFFFFFu && s_res[2] > (uint32_t)cap) bc += 1;  // suffix(bc + 1) < kloc <= cap
    {
        uint64_t* cand = p.cand + ((int64_t)qi * p.max_chunks + cidx) * cap;
        uint32_t n_cand = 0;
        for (int base = 0; base < n; base += kScanThreads * kTailPer) {
            const int first = base + warp * 32 * kTailPer + lane;
            uint64_t v[kTailPer];
            bool keep[kTailPer];
#pragma unroll
            for (int u = 0; u < kTailPer; ++u) {
                const int i = first + u * 32;
                const uint32_t key = i < n ? float_key(ssc[i]) : 0u;
                keep[u] = i < n && (key >> (32 - kKeyBits)) >= bc;
                v[u] = composite(key, c0 + i);
            }
            n_cand += compact_round<kScanThreads, kTailPer>(
                v, keep, n_cand, [&](uint32_t pos, uint64_t x) { if (pos < (uint32_t)cap) cand[pos] = x; }, s_wsum);
        }
        if (tid == 0) p.meta[(int64_t)qi * p.max_chunks + cidx] = (bc << 16) | n_cand;
    }
}

// ---- final selection (decode / standalone path) -------------------------------------------------
//
// One thread-block cluster of kFinalF CTAs per query, after the scan grid.  Every CTA derives the
// threshold bin b1 from the query's histogram (the k-th largest key lies in bin b1; the entries of
// bins >= b1, n_tot of them, are exactly the ones to consider), then gathers those members from
// its share of the chunks, in index order: from a chunk's candidates when b_c <= b1 (they hold all
// of its members), else from its stored scores.  It publishes its count in the leader (rank 0);
// after a cluster barrier each CTA stores its members at its offset of the leader's list
// (distributed shared memory, or the global segment buffer for a list longer than shared memory
// holds); after a second barrier the leader radix-selects the exact threshold inside bin b1 (64-bit
// key: score key << 32 | ~index, unique, ties to the lower index) and compacts the k indices in
// ascending order.
constexpr int kFinalF = 8;           // CTAs per query
constexpr int kFinalThreads = 256;
constexpr int kFinalDynSmem = kListKeys * 8;  // the members list (also this CTA's chunk words)
constexpr int kFinalChunks = (kKeyBins - 2) / 2;  // chunks per CTA whose words fit the histogram's space

__global__ void __launch_bounds__(kFinalThreads, 1) index_final_kernel(IndexParams p) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ __align__(16) uint32_t hist[kKeyBins];
    __shared__ uint32_t s_wsum[kFinalThreads / 32];
    __shared__ uint32_t s_res[4];
    __shared__ uint32_t s_cnt[kFinalF];  // the leader's: members per rank
    __shared__ uint32_t s_tot;
    grid_dep_wait();  // the scan's histograms, candidates and scores
    grid_dep_launch();
    const int qi = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_ctarank();
    const csa_query qr = p.queries[qi];
    const bool seq_ok = qr.seq >= 0 && qr.reserved == 0;
    const csa_seq sq = seq_ok ? p.seqs[qr.seq] : csa_seq{0, 0, 0, 0};
    const bool valid = seq_ok && qr.len >= 1 && qr.len <= sq.len;
    const int64_t E = valid ? qr.len / p.m : 0;
    // the scan handled (and reported) these; the outcome is uniform over the cluster
    if (!valid || E > p.max_entries || E <= p.k) {
        if (rank == 0 && tid == 0) signal_ready(p, qi);
        return;
    }
    const int64_t chunk = p.chunk;
    const int nch = (int)((E + chunk - 1) / chunk);
    const int cap = p.cand_cap;
    const int cb = (int)((int64_t)nch * rank / kFinalF), ce = (int)((int64_t)nch * (rank + 1) / kFinalF);
    const int nmine = ce - cb;
    const uint32_t* meta = p.meta + (int64_t)qi * p.max_chunks + cb;
    const bool words_smem = nmine <= kFinalChunks;
    // 1. the threshold bin; the histogram and this CTA's chunk words are loaded together
    uint32_t* mw = reinterpret_cast<uint32_t*>(dsm);
    {
        const uint32_t* gh = p.hist + (int64_t)qi * kKeyBins;
        uint32_t hv[kKeyBins / kFinalThreads];
#pragma unroll
        for (int i = 0; i < kKeyBins / kFinalThreads; ++i) hv[i] = __ldcg(gh + tid + i * kFinalThreads);
        if (words_smem)
            for (int c = tid; c < nmine; c += kFinalThreads) mw[c] = __ldcg(meta + c);
#pragma unroll
        for (int i = 0; i < kKeyBins / kFinalThreads; ++i) hist[tid + i * kFinalThreads] = hv[i];
    }
    __syncthreads();
    find_bin<kFinalThreads, kKeyBins>(hist, (uint32_t)p.k, s_wsum, s_res);
    const uint32_t b1 = s_res[0], above = s_res[1], at = s_res[2];
    if (b1 == 0xFFFFFFFFu) {  // the histogram holds fewer than k scores: cannot happen for E > k
        if (tid == 0 && rank == 0) {
            report(p.status, CSA_ERR_INDEX);
            signal_ready(p, qi);
        }
        return;
    }
    const uint32_t n_bin = at - above, need = (uint32_t)p.k - above, n_tot = at;
    const bool in_smem = n_tot <= (uint32_t)kListKeys;
    // 2. this CTA's source items, numbered densely chunk after chunk: src[c] = the first number of
    //    chunk cb + c (src[nmine] = the total), flag[c] = its members come from its candidates; in
    //    the histogram's space (free until the radix select), or the global chunk words
    uint32_t* src = words_smem ? hist : p.coff + (int64_t)qi * (p.max_chunks + kFinalF) + cb + rank;
    uint32_t* flag = hist + kFinalChunks + 1;
    {
        uint32_t carry = 0;
        for (int c0 = 0; c0 < nmine; c0 += kFinalThreads) {
            const int c = c0 + tid;
            uint32_t len = 0, fc = 0;
            if (c < nmine) {
                const uint32_t w = words_smem ? mw[c] : __ldcg(meta + c);
                fc = (w >> 16) <= b1 ? 1u : 0u;
                const int64_t cc = cb + c;
                len = fc ? (w & 0xFFFFu) : (uint32_t)(min(E, (cc + 1) * chunk) - cc * chunk);
            }
            uint32_t tot;
            const uint32_t ex = excl_scan<kFinalThreads>(len, s_wsum, &tot);  // synchronizes: mw reads done
            if (c < nmine) {
                src[c] = carry + ex;
                if (words_smem) flag[c] = fc;
            }
            carry += tot;
        }
        if (tid == 0) {
            src[nmine] = carry;
            s_tot = carry;
        }
    }
    if (!words_smem) __threadfence_block();
    __syncthreads();
    const uint32_t S = s_tot;
    auto src_at = [&](int c) -> uint32_t { return words_smem ? src[c] : __ldcg(src + c); };
    auto from_cand = [&](int c) -> bool { return words_smem ? flag[c] != 0u : (__ldcg(meta + c) >> 16) <= b1; };
    const unsigned long long* cand_q =
        reinterpret_cast<const unsigned long long*>(p.cand) + ((int64_t)qi * p.max_chunks + cb) * cap;
    const float* srow_q = p.scores + (int64_t)qi * p.e_stride;
    uint64_t* lst = reinterpret_cast<uint64_t*>(dsm);  // this CTA's members; the leader's: the whole list
    uint64_t* gseg = p.seg + (int64_t)qi * p.e_seg;
    // One pass over the source items in rounds of kTailPer per thread, laid out warp-contiguously
    // (see compact_round).  All addresses of a round are found first (chunk boundaries from shared
    // memory), then the loads are issued unconditionally, back to back, so a round costs one memory
    // latency (a load inside the data-dependent branches would be consumed at their join, one
    // latency per item).  An item of a stored-score chunk loads the aligned 8-byte word holding its
    // score (a word reaching 4 bytes past the score rows stays inside the workspace: the segment
    // buffer follows them).  Members are handed to sink(position among this CTA's members, key).
    auto gather = [&](auto&& sink) -> uint32_t {
        uint32_t written = 0;
        for (uint32_t base = 0; base < S; base += kFinalThreads * kTailPer) {
            const uint32_t first = base + (uint32_t)(warp * 32 * kTailPer + lane);
            int c = 0;
            if (first < S) {  // the chunk holding item `first`: the last c with src[c] <= first
                int lo = 0, hi = nmine - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (src_at(mid) <= first) lo = mid; else hi = mid - 1;
                }
                c = lo;
            }
            const unsigned long long* ad[kTailPer];
            uint32_t jk[kTailPer];  // bit 31: a stored score, bit 30: in the high half of its word; bits 0..29: j
            uint32_t c_lo = first < S ? src_at(c) : 0u, c_hi = first < S ? src_at(c + 1) : 0u;
            bool fcand = first < S && from_cand(c);
#pragma unroll
            for (int u = 0; u < kTailPer; ++u) {
                const uint32_t i = first + u * 32;
                ad[u] = cand_q;  // a valid address for an empty slot
                jk[u] = 0u;
                if (i < S) {
                    while (i >= c_hi) {  // next chunk with items
                        ++c;
                        c_lo = c_hi;
                        c_hi = src_at(c + 1);
                        fcand = from_cand(c);
                    }
                    const uint32_t slot = i - c_lo;
                    if (fcand) {
                        ad[u] = cand_q + (int64_t)c * cap + slot;
                    } else {
                        const uint32_t j = (uint32_t)((int64_t)(cb + c) * chunk + slot);
                        const uintptr_t f = reinterpret_cast<uintptr_t>(srow_q + j);
                        ad[u] = reinterpret_cast<const unsigned long long*>(f & ~(uintptr_t)7);
                        jk[u] = 0x80000000u | ((f & 4) ? 0x40000000u : 0u) | j;
                    }
                }
            }
            uint64_t v[kTailPer];
#pragma unroll
            for (int u = 0; u < kTailPer; ++u) v[u] = __ldcg(ad[u]);
            bool keep[kTailPer];
#pragma unroll
            for (int u = 0; u < kTailPer; ++u) {
                if (jk[u] & 0x80000000u) {
                    const uint32_t w = (jk[u] & 0x40000000u) ? (uint32_t)(v[u] >> 32) : (uint32_t)v[u];
                    v[u] = composite(float_key(__uint_as_float(w)), jk[u] & 0x3FFFFFFFu);
                }
                keep[u] = first + u * 32 < S && (uint32_t)(v[u] >> (64 - kKeyBits)) >= b1;
            }
            written += compact_round<kFinalThreads, kTailPer>(v, keep, written, sink, s_wsum);
        }
        return written;
    };
    // 3. members into the list: kept in this CTA's shared memory first (a list that fits), counts to
    //    the leader, then every CTA stores its members at its offset of the leader's list
    const uint32_t n_mine = gather([&](uint32_t pos, uint64_t x) {
        if (in_smem && pos < (uint32_t)kListKeys) lst[pos] = x;
    });
    if (tid == 0) st_cluster_u32(&s_cnt[rank], 0, n_mine);
    cluster_barrier();
    uint32_t off, total;  // members of the ranks before this one, of all ranks
    {
        const uint32_t cr = lane < kFinalF ? ld_cluster_u32(&s_cnt[lane], 0) : 0u;
        off = (uint32_t)lane < rank ? cr : 0u;
        total = cr;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            off += __shfl_xor_sync(0xffffffffu, off, o);
            total += __shfl_xor_sync(0xffffffffu, total, o);
        }
    }
    if (total != n_tot) {  // the members must be exactly the histogram's count of bins >= b1
        if (tid == 0 && rank == 0) {
            report(p.status, CSA_ERR_INDEX);
            signal_ready(p, qi);
        }
        cluster_barrier();  // every CTA takes the same barriers
        return;
    }
    if (in_smem) {
        if (rank != 0)
            for (uint32_t i = tid; i < n_mine; i += kFinalThreads) st_cluster_u64(&lst[off + i], 0, lst[i]);
    } else {
        gather([&](uint32_t pos, uint64_t x) { gseg[off + pos] = x; });
    }
    cluster_barrier();  // the leader's list is complete
    int32_t* out = p.idx_out + (int64_t)qi * p.k;
    if (rank == 0) {
        // 4. the exact threshold inside bin b1, then compaction in index order
        const KeyList L{in_smem ? lst : nullptr, in_smem ? nullptr : gseg};
        const uint64_t T = need == n_bin ? ((uint64_t)b1 << (64 - kKeyBits)) : radix_select<kFinalThreads, kKeyBits>(L, n_tot, need, b1, hist,
                                                                                               s_wsum, s_res);
        float* sout = p.score_out ? p.score_out + (int64_t)qi * p.k : nullptr;
        uint32_t kept = 0;
        for (uint32_t base = 0; base < n_tot; base += kFinalThreads * kTailPer) {
            const uint32_t first = base + (uint32_t)(warp * 32 * kTailPer + lane);
            uint64_t v[kTailPer];
            bool keep[kTailPer];
#pragma unroll
            for (int u = 0; u < kTailPer; ++u) {
                const uint32_t i = first + u * 32;
                v[u] = i < n_tot ? L.get(i) : 0ull;
                keep[u] = i < n_tot && v[u] >= T;
            }
            kept += compact_round<kFinalThreads, kTailPer>(v, keep, kept, [&](uint32_t o, uint64_t x) {
                if (o < (uint32_t)p.k) {
                    out[o] = (int32_t)(0xFFFFFFFFu - (uint32_t)(x & 0xFFFFFFFFull));
                    if (sout) sout[o] = key_float((uint32_t)(x >> 32));
                }
            }, s_wsum);
        }
        if (tid == 0 && kept != (uint32_t)p.k) report(p.status, CSA_ERR_INDEX);
        if (p.ready) {
            __syncthreads();  // every index store of the CTA precedes the release
            if (tid == 0) signal_ready(p, qi);
        }
    }
    if (!p.prefetch_rows) return;  // (uniform over the cluster)
    cluster_barrier();  // the indices are out (the barrier orders global memory at cluster scope)
    // 5. the attention that follows gathers the selected rows: every CTA of the cluster starts
    //    bringing its share of them into L2
    for (int o = (int)rank * kFinalThreads + tid; o < p.k; o += kFinalF * kFinalThreads) {
        const int32_t j = __ldcg(out + o);
        if (j >= 0) prefetch_l2(p.prefetch_rows + (sq.csa_off + j) * p.prefetch_row_bytes, p.prefetch_row_bytes);
    }
}
// FP4 copies (E2M1 codes, 32-channel power-of-two block scales; quant_mx4) of the stored bf16 entries
// [ranges[b][0], ranges[b][1]) of every sequence's CSA cache (which = 0, ratio m) or HCA cache
// (which = 1, ratio m_hca): d / 8 threads per entry, four lanes per block.
__global__ void __launch_bounds__(256) quantize_entries_kernel(const csa_seq* seqs, const int64_t* ranges, int which,
                                                               int ratio, int d, const uint16_t* entries,
                                                               uint8_t* entries_q, uint8_t* scales, int* status) {
    const int b = blockIdx.y;
    const int tpe = d / 8;  // threads per entry (a multiple of 4)
    const int64_t e0 = ranges[2 * b], e1 = ranges[2 * b + 1];
    const csa_seq sq = seqs[b];
    if (e0 < 0 || e1 < e0 || (int64_t)ratio * e1 > sq.len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(status, CSA_ERR_INDEX);
        return;
    }
    const int lane = threadIdx.x & 31, sub = threadIdx.x / tpe, g = threadIdx.x % tpe;
    const unsigned mask = 0xFu << (lane & ~3);
    const int64_t base = which ? sq.hca_off : sq.csa_off;
    for (int64_t j = e0 + (int64_t)blockIdx.x * (256 / tpe) + sub; j < e1; j += (int64_t)gridDim.x * (256 / tpe)) {
        const int64_t row = base + j;
        const uint4 v = *reinterpret_cast<const uint4*>(entries + row * d + 8 * g);
        uint32_t sb;
        const uint32_t q = quant_mx4(v, mask, &sb);
        *reinterpret_cast<uint32_t*>(entries_q + row * (d / 2) + 4 * g) = q;
        if ((g & 3) == 0) scales[row * (d / 32) + g / 4] = (uint8_t)sb;
    }
}

constexpr size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

namespace {

// Scan chunking of Q queries of up to e_stride entries: chunks of a multiple of 64 entries sized so
// that all chunks make about one wave of two scan CTAs per SM (so SMs carry equal shares), at least
// 256 and at most what the chunk's score buffer in shared memory holds.  Two CTAs, not more: a pass
// keeps its sixteen 16-byte key loads per thread in registers (up to 128 per thread), and the
// loads in flight, not the warp count, set the streaming rate.
struct ScanPlan {
    int64_t chunk;
    int max_chunks;
    int cap;
};

ScanPlan scan_plan(int Q, int64_t e_stride) {
    constexpr int64_t kSlots = 148 * 2;
    ScanPlan sp;
    int64_t c = (e_stride * Q + kSlots - 1) / kSlots;
    c = ((c + 63) / 64) * 64;
    if (c < 256) c = 256;
    if (c > kScanChunkMax) c = kScanChunkMax;
    sp.chunk = c;
    sp.max_chunks = (int)((e_stride + c - 1) / c);
    sp.cap = (int)(c / 4 < 256 ? c / 4 : 256);
    return sp;
}

// Per-chunk words and candidate keys are sized by bounds that hold for every chunk size the plan
// can choose (chunks of at least 256 entries keeping at most a quarter of their entries, at most
// 256), so the workspace of Q queries also serves any smaller query count.  A query's chunk words
// hold max_chunks + kFinalF entries (the final select's prefix over a CTA's chunks has one more,
// per CTA).
size_t chunk_words(int Q, int64_t e_stride) { return (size_t)Q * (size_t)(e_stride / 256 + 1 + kFinalF); }
size_t cand_keys(int Q, int64_t e_stride) { return (size_t)Q * (size_t)(e_stride / 4 + 256); }

}  // namespace

size_t index_zero_bytes(int Q) { return align256((size_t)Q * (kKeyBins + 6) * 4); }

uint32_t* index_ready_words(void* ws, int Q) { return static_cast<uint32_t*>(ws) + (size_t)Q * kKeyBins; }

size_t index_ws_bytes(int Q, int64_t e_stride) {
    size_t s = index_zero_bytes(Q);
    s += align256((size_t)Q * e_stride * 4);
    s += align256((size_t)Q * (e_stride + kSegPad) * 8);
    s += 2 * align256(chunk_words(Q, e_stride) * 4);
    s += align256(cand_keys(Q, e_stride) * 8);
    return s;
}

void index_ws_carve(IndexParams& p, void* ws, int Q, int64_t e_stride) {
    const ScanPlan sp = scan_plan(Q, e_stride);
    char* b = static_cast<char*>(ws);
    p.hist = reinterpret_cast<uint32_t*>(b);
    b += index_zero_bytes(Q);
    p.scores = reinterpret_cast<float*>(b);
    b += align256((size_t)Q * e_stride * 4);
    p.seg = reinterpret_cast<uint64_t*>(b);
    b += align256((size_t)Q * (e_stride + kSegPad) * 8);
    p.meta = reinterpret_cast<uint32_t*>(b);
    b += align256(chunk_words(Q, e_stride) * 4);
    p.coff = reinterpret_cast<uint32_t*>(b);
    b += align256(chunk_words(Q, e_stride) * 4);
    p.cand = reinterpret_cast<uint64_t*>(b);
    p.ready = nullptr;
    p.debug_fault = 0;
    p.qsync = nullptr;
    p.sms = 0;
    p.e_stride = e_stride;
    p.e_seg = e_stride + kSegPad;
    p.chunk = sp.chunk;
    p.max_chunks = sp.max_chunks;
    p.cand_cap = sp.cap;
}

cudaError_t launch_index_topk(IndexParams& p, int64_t max_entries, cudaStream_t stream, bool zero_ws,
                              cudaEvent_t mid, bool pdl, bool sampled) {
    if (sampled) {
        // scores are already in p.scores; one select CTA per query holds its whole row
        if (max_entries > kSelBufMax) return cudaErrorInvalidValue;
        const int64_t buf = ((max_entries + 3) / 4) * 4;
        const size_t smem = SelSmem::bytes(buf < 4 ? 4 : buf);
        static PerDeviceOnce attr;
        cudaError_t e = attr.run([] {
            return cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SelSmem::bytes(kSelBufMax));
        });
        if (e != cudaSuccess) return e;
        return launch_kernel(index_select_kernel, dim3((unsigned)p.Q), dim3(kSelectThreads), smem, stream, pdl, p);
    }
    if (zero_ws) {
        // the histograms sit at the start of the workspace
        cudaError_t e = cudaMemsetAsync(p.hist, 0, index_zero_bytes(p.Q), stream);
        if (e != cudaSuccess) return e;
    }
    // the scan's final select packs entry indices into 30 bits
    if (max_entries >= (int64_t(1) << 30)) return cudaErrorInvalidValue;
    cudaError_t e;
    // chunk 0 of a query that selects all of its entries writes the result alone
    const int64_t gx = max_entries > p.k ? (max_entries + p.chunk - 1) / p.chunk : 1;
    if (gx > p.max_chunks) return cudaErrorInvalidValue;  // the workspace was carved for fewer entries
    const dim3 grid((unsigned)gx, (unsigned)p.Q);
    const bool dep = pdl && !zero_ws;
    // the scan grid selects itself when all of its CTAs fit the SMs at once (two per SM)
    const bool fused = p.qsync && p.sms > 0 && gx * (int64_t)p.Q <= 2 * (int64_t)p.sms;
    if (!fused) p.qsync = nullptr;
    // with the key histogram in static shared memory, the dynamic part needs the opt-in (per device)
    static PerDeviceOnce attr_scan;
    e = attr_scan.run([] {
        cudaError_t r = cudaSuccess;
        for (auto f : {index_scan_kernel<1, false>, index_scan_kernel<2, false>, index_scan_kernel<1, true>,
                       index_scan_kernel<2, true>})
            if (r == cudaSuccess) r = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kScanDynSmem);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(index_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFinalDynSmem);
        return r;
    });
    if (e != cudaSuccess) return e;
    if (p.keys_q)
        e = p.d_I == 64 ? launch_kernel(index_scan_kernel<2, true>, grid, dim3(kScanThreads), kScanDynSmem, stream, dep, p)
                        : launch_kernel(index_scan_kernel<1, true>, grid, dim3(kScanThreads), kScanDynSmem, stream, dep, p);
    else
        e = p.d_I == 64 ? launch_kernel(index_scan_kernel<2, false>, grid, dim3(kScanThreads), kScanDynSmem, stream, dep, p)
                        : launch_kernel(index_scan_kernel<1, false>, grid, dim3(kScanThreads), kScanDynSmem, stream, dep, p);
    if (e != cudaSuccess) return e;
    if (mid && (e = cudaEventRecordWithFlags(mid, stream, cudaEventRecordExternal)) != cudaSuccess) return e;
    if (fused) return cudaSuccess;
    // the exact selection: one cluster of kFinalF CTAs per query
    return launch_kernel_cluster(index_final_kernel, dim3(kFinalF, (unsigned)p.Q), dim3(kFinalThreads), kFinalDynSmem,
                                 stream, pdl, dim3(kFinalF, 1, 1), p);
}

cudaError_t launch_quantize_entries(const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries, int which,
                                    int ratio, int d, const uint16_t* entries, uint8_t* entries_q, uint8_t* scales,
                                    int* status, cudaStream_t stream) {
    if (max_entries <= 0) return cudaSuccess;
    const int per_cta = 256 / (d / 8);
    int64_t gx = (max_entries + per_cta - 1) / per_cta;
    if (gx > 8192) gx = 8192;
    quantize_entries_kernel<<<dim3((unsigned)gx, (unsigned)B), 256, 0, stream>>>(seqs, ranges, which, ratio, d, entries,
                                                                                entries_q, scales, status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_keys(const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries, int m,
                                 int d_I, const uint16_t* keys, uint8_t* keys_q, uint8_t* scales, int* status,
                                 cudaStream_t stream) {
    if (max_entries <= 0) return cudaSuccess;
    const int per_cta = 256 / (d_I / 8);
    int64_t gx = (max_entries + per_cta - 1) / per_cta;
    if (gx > 8192) gx = 8192;
    quantize_keys_kernel<<<dim3((unsigned)gx, (unsigned)B), 256, 0, stream>>>(seqs, ranges, m, d_I, keys, keys_q,
                                                                             scales, status);
    return cudaGetLastError();
}

}  // namespace csa

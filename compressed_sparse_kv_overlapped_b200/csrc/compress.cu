// compress.cu -- a1/a2: the token-axis softmax compressor, full-pass kernels.
//
// "DeepSeek V4 comprimeix el context: aixi funcionen CSA i HCA", sections "DeepSeek comprimeix la
// dimensio temporal" (an entry is a softmax-weighted sum of the tokens it summarises, with a
// separate weight per channel) and "Finestres solapades per evitar fronteres artificials"
// (overlapping windows, weights recomputed per window); "Frontier Techniques: NTK RoPE, CSA+HCA,
// QAT, MTP", 2.1 (m = 4) and 2.2 (m' = 128).
//
// compress_tile_kernel (CSA ratio 4, HCA ratio a power of two up to 128): one CTA per (128-token
// tile, sequence, 64-channel slice).  One thread issues four TMA boxes of 132 rows (the tile plus
// the 4-token halo the first CSA window reaches back to) of the latent, both logit arrays and the
// indexer keys into shared memory, so every token row is read from HBM once for both caches.
// Thread (u, g) (u = 4-token block 0..31, g = 8-channel group 0..7) then builds CSA entry 32*tile + u
// from the two 4-token softmax partials of its window and the partial of block u for HCA, whose
// entries are merged by the block tree of compress_dev.cuh.  Entries are stored as bf16 with 16-byte
// stores.  The window arithmetic is shared with the decode append (identical entries).
//
// compress_kernel (other ratios): one thread per 8 channels of one entry, an online softmax over
// the window read with coalesced 16-byte loads.
#include <cstring>

#include "compress_dev.cuh"
#include "kernels.h"
#include "tma.h"

namespace csa {

namespace {

__global__ void __launch_bounds__(256) compress_kernel(CompressParams p) {
    const int b = blockIdx.y;
    const csa_seq sq = p.seqs[b];
    const int64_t r0 = p.ranges ? p.ranges[2 * b] : p.range_begin;
    const int64_t r1 = p.ranges ? p.ranges[2 * b + 1] : p.range_end;
    const int64_t e0 = p.token_ranges ? r0 / p.m : r0, e1 = p.token_ranges ? r1 / p.m : r1;
    if (r0 < 0 || r1 < r0 || (int64_t)p.m * e1 > sq.len || (p.token_ranges && r1 > sq.len)) {
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

constexpr int kTileTok = 128;                  // tokens per tile: one 128-token HCA block, 32 CSA entries
static_assert(hca_block_shape(kTileTok) && !hca_block_shape(2 * kTileTok), "HCA blocks divide a tile");
constexpr int kHalo = 4;                       // the previous CSA block (window of the tile's first entry)
constexpr int kBoxRows = kTileTok + kHalo;     // rows of every TMA box
constexpr int kSlice = 64;                     // channels per CTA
constexpr int kBoxBytes = kBoxRows * kSlice * 2;

struct TileMaps {
    CUtensorMap x, lc, lh, ki;
};

struct TileSmem {
    static constexpr int kX = 0;
    static constexpr int kLc = kX + kBoxBytes;
    static constexpr int kLh = kLc + kBoxBytes;
    static constexpr int kKi = kLh + kBoxBytes;       // d_I * 2 bytes per row (at most 128)
    static constexpr int kXs = kKi + kBoxBytes;       // HCA tree exchange: 8 warps x 8 groups x 24 floats
    static constexpr int kSs = kXs + 8 * 8 * 24 * 4;  // per-entry sums of squares (normalization): 64 floats
    static constexpr int kBar = kSs + 64 * 4;
    static constexpr int kTotal = kBar + 16;
    static constexpr int kAlloc = kTotal + 128;       // slack for 128-byte alignment
};

__global__ void __launch_bounds__(256, 3) compress_tile_kernel(const __grid_constant__ TileMaps maps,
                                                                TileCompressParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + TileSmem::kBar);
    float* xs = reinterpret_cast<float*>(sm + TileSmem::kXs);
    const int b = blockIdx.y, slice = blockIdx.z;
    const int tid = threadIdx.x, u = tid >> 3, g = tid & 7;
    const csa_seq sq = p.seqs[b];
    const int64_t r0 = p.ranges ? p.ranges[2 * b] : p.range_begin;
    const int64_t r1 = p.ranges ? p.ranges[2 * b + 1] : p.range_end;
    // the entries this call writes for sequence b: CSA [cj0, cj1), HCA [hh0, hh1)
    int64_t cj0 = 0, cj1 = 0, hh0 = 0, hh1 = 0, t_first;
    const int mh = p.m_hca;
    if (p.range_kind == 0) {
        cj0 = r0; cj1 = r1; t_first = 4 * r0;
    } else if (p.range_kind == 1) {
        hh0 = r0; hh1 = r1; t_first = mh * r0;
    } else {
        if (p.do_csa) { cj0 = r0 / 4; cj1 = r1 / 4; }
        if (p.do_hca) { hh0 = r0 / mh; hh1 = r1 / mh; }
        t_first = r0;
    }
    if (r0 < 0 || r1 < r0 || 4 * cj1 > sq.len || (int64_t)mh * hh1 > sq.len || (p.range_kind == 2 && r1 > sq.len) ||
        sq.tok_off + t_first + (int64_t)kTileTok * gridDim.x + kBoxRows > 0x7FFFFFFF) {
        if (tid == 0 && blockIdx.x == 0 && slice == 0) report(p.status, CSA_ERR_INDEX);
        return;
    }
    const int64_t tile = t_first / kTileTok + blockIdx.x;
    const int64_t tt0 = tile * kTileTok;  // first token of the tile
    // this tile's share
    const int64_t c_lo = max(cj0, tt0 / 4), c_hi = min(cj1, (tt0 + kTileTok) / 4);
    const int64_t h_lo = max(hh0, tt0 / mh), h_hi = min(hh1, (tt0 + kTileTok) / mh);
    const bool csa = p.do_csa && c_lo < c_hi;
    const bool hca = p.do_hca && h_lo < h_hi;
    if (!csa && !hca) return;
    // once any CTA has given up on a wait, later CTAs do no work (bounded total time on a fault); not
    // with normalization, where the CTAs of a cluster must all reach its barriers
    if (!p.norm_c && !p.norm_h && p.status && *reinterpret_cast<volatile int*>(p.status) == CSA_ERR_TIMEOUT)
        return;
    // rows [box0, box0 + kBoxRows) of the sequence cover every token the tile's entries use and end at
    // the last token used, so no row past the sequence's valid rows is read (negative rows read 0)
    const int64_t t_hi = max(csa ? 4 * c_hi : 0, hca ? (int64_t)mh * h_hi : 0);
    int64_t box0 = tt0 - kHalo;
    if (box0 + kBoxRows > t_hi) box0 = t_hi - kBoxRows;
    const bool keys = csa && p.do_keys && slice * kSlice < p.d_I;
    const int d = p.d;
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        const uint32_t bytes = (uint32_t)kBoxBytes * (1u + (csa ? 1u : 0u) + (hca ? 1u : 0u)) +
                               (keys ? (uint32_t)(kBoxRows * p.d_I * 2) : 0u);
        mbar_arrive_expect_tx(bar, bytes);
        const int y = (int)(sq.tok_off + box0);
        const uint32_t s0 = smem_u32(sm);
        tma_load_2d(s0 + TileSmem::kX, &maps.x, slice * kSlice, y, bar);
        if (csa) tma_load_2d(s0 + TileSmem::kLc, &maps.lc, slice * kSlice, y, bar);
        if (hca) tma_load_2d(s0 + TileSmem::kLh, &maps.lh, slice * kSlice, y, bar);
        if (keys) tma_load_2d(s0 + TileSmem::kKi, &maps.ki, 0, y, bar);
    }
    __syncthreads();
    // the outcome is made CTA-uniform, so a timeout (recorded; nothing is written) never leaves some
    // threads at a barrier below without the others
    const bool norm = p.norm_c || p.norm_h;  // entry normalization: the slices exchange partial sums
    const bool loaded = __syncthreads_and(mbar_wait(bar, 0, p.status, nullptr) ? 1 : 0) != 0;
    // a timeout is recorded and nothing is written; with normalization the CTA still takes the
    // cluster barriers below, which every CTA of the cluster must reach
    if (!loaded && !norm) return;

    const uint16_t* sx = reinterpret_cast<const uint16_t*>(sm + TileSmem::kX);
    const uint16_t* slc = reinterpret_cast<const uint16_t*>(sm + TileSmem::kLc);
    const uint16_t* slh = reinterpret_cast<const uint16_t*>(sm + TileSmem::kLh);
    const uint16_t* ski = reinterpret_cast<const uint16_t*>(sm + TileSmem::kKi);
    float* ss_c = reinterpret_cast<float*>(sm + TileSmem::kSs);       // [32] CSA entries of the tile
    float* ss_h = ss_c + 32;                                          // [32] HCA entries of the tile
    const int c0 = slice * kSlice + g * 8;  // this thread's first channel
    const int lane = tid & 31;

    const int64_t j = tt0 / 4 + u;
    const bool c_mine = loaded && csa && j >= c_lo && j < c_hi;
    float cv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c_mine) {
        const int rbase = (int)(4 * j - 4 - box0);  // smem row of window position 0
        auto fetch = [&](int tensor, int pos) -> uint4 {
            const int r = rbase + pos;
            const uint16_t* base = tensor == 0 ? slc : tensor == 1 ? sx : ski;
            const int stride = tensor == 2 ? p.d_I : kSlice;
            return *reinterpret_cast<const uint4*>(base + r * stride + g * 8);
        };
        if (keys && c0 < p.d_I) {
            uint4 key;
            csa_entry_block4<true>(j, d, p.bias_c + c0, fetch, cv, &key);
            *reinterpret_cast<uint4*>(p.entry_keys + (sq.csa_off + j) * p.d_I + c0) = key;
        } else {
            csa_entry_block4<false>(j, d, p.bias_c + c0, fetch, cv, nullptr);
        }
    }
    // HCA: m' >= 16 in the 16-tokens-per-warp form (lane = channel pair); m' = 4, 8 in the 4-token
    // block form (the block tree)
    const bool h16 = mh >= 16;
    float hv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    Part2 H2;
    bool h_mine = false;
    int64_t h = 0;
    if (hca && h16) {
        const int w16 = tid >> 5;
        int r = (int)(tt0 + 16 * w16 - box0);  // smem row of the warp's first token
        if (r < 0 || r + 16 > kBoxRows) r = 0;  // tokens past the loaded rows belong to no entry written here
        const int cp = slice * kSlice + 2 * lane;
        auto fetch = [&](int tensor, int t) -> uint32_t {
            const uint16_t* base = tensor == 0 ? slh : sx;
            return *reinterpret_cast<const uint32_t*>(base + (r + t) * kSlice + 2 * lane);
        };
        const int brow0 = (16 * w16) & (mh - 1);
        auto bias2 = [&](int t) -> float2 {
            return __ldg(reinterpret_cast<const float2*>(p.bias_h + (int64_t)(brow0 + t) * d + cp));
        };
        hca_part16(fetch, bias2, H2);
        hca_merge_warps(H2, mh / 16, xs);
        h = (tt0 + 16 * w16) / mh;
        h_mine = loaded && (w16 % (mh / 16)) == 0 && h >= h_lo && h < h_hi;
        hv[0] = entry_div(H2.acc[0], H2.den[0]);
        hv[1] = entry_div(H2.acc[1], H2.den[1]);
    } else if (hca) {
        const int nb = mh / 4;  // blocks per HCA entry
        // block u's 4 tokens; blocks past the loaded rows belong to no entry this tile writes
        int r = (int)(tt0 + 4 * u - box0);
        if (r < 0 || r + 4 > kBoxRows) r = 0;
        uint4 lg[4], xv[4], kv[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            lg[t] = *reinterpret_cast<const uint4*>(slh + (r + t) * kSlice + g * 8);
            xv[t] = *reinterpret_cast<const uint4*>(sx + (r + t) * kSlice + g * 8);
            kv[t] = make_uint4(0, 0, 0, 0);
        }
        Part8 P;
        part4<false>(lg, xv, kv, p.bias_h + (int64_t)((4 * u) & (mh - 1)) * d + c0, d, P);
        hca_tree(P, nb, xs);
        h = (tt0 + 4 * u) / mh;
        const bool holder = (u & (nb - 1)) == 0 && (nb < 8 || lane < 8);
        h_mine = loaded && holder && h >= h_lo && h < h_hi;
#pragma unroll
        for (int i = 0; i < 8; ++i) hv[i] = entry_div(P.acc[i], P.den[i]);
    }
    float inv_c = 1.f, inv_h = 1.f;
    if (norm) {
        // partial sums of squares over this CTA's 64 channels, one per entry of the tile, then the
        // totals over the cluster's slices
        const float sc = sum_lane8(sumsq8(cv));
        const float sh = h16 ? warp_sum(__fmaf_rn(hv[1], hv[1], __fmaf_rn(hv[0], hv[0], 0.f))) : sum_lane8(sumsq8(hv));
        if (g == 0) ss_c[u] = sc;
        if (h_mine && (h16 ? lane == 0 : g == 0)) ss_h[h - tt0 / mh] = sh;
        cluster_barrier();
        const int ns = (int)gridDim.z;
        if (c_mine && p.norm_c) inv_c = rms_inv(cluster_sum(ss_c + u, ns), d, p.eps);
        if (h_mine && p.norm_h) inv_h = rms_inv(cluster_sum(ss_h + (h - tt0 / mh), ns), d, p.eps);
        cluster_barrier();  // no CTA leaves while another still reads its shared memory
    }
    if (c_mine)
        *reinterpret_cast<uint4*>(p.entries + (sq.csa_off + j) * d + c0) = entry_bf16(cv, p.norm_c ? p.norm_c + c0 : nullptr, inv_c);
    if (h_mine) {
        if (h16) {
            const int cp = slice * kSlice + 2 * lane;
            *reinterpret_cast<uint32_t*>(p.hca_entries + (sq.hca_off + h) * d + cp) =
                entry_bf16x2(hv[0], hv[1], p.norm_h ? p.norm_h + cp : nullptr, inv_h);
        } else {
            *reinterpret_cast<uint4*>(p.hca_entries + (sq.hca_off + h) * d + c0) =
                entry_bf16(hv, p.norm_h ? p.norm_h + c0 : nullptr, inv_h);
        }
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

cudaError_t launch_compress_tiles(const TileCompressParams& p, int64_t max_span, cudaStream_t stream) {
    if (max_span <= 0 || (!p.do_csa && !p.do_hca)) return cudaSuccess;
    if (p.d % kSlice != 0 || (p.d_I != 32 && p.d_I != 64) || (p.do_hca && !hca_block_shape(p.m_hca)))
        return cudaErrorInvalidValue;
    static PerDeviceOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(compress_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    TileSmem::kAlloc);
    });
    if (e != cudaSuccess) return e;
    // tensor maps over the raw arrays; boxes of 132 rows x 64 channels (the indexer keys: all d_I
    // channels), no swizzle.  The row extent is left open: the kernel starts every box inside the
    // sequence's valid rows or before row 0, where the box reads zeros.
    TileMaps maps;
    std::memset(&maps, 0, sizeof maps);
    const uint64_t rows = 0x7FFFFFFFull;
    e = tensor_map_2d_bf16(&maps.x, p.x, p.d, rows, (uint64_t)p.d * 2, kSlice, kBoxRows, false);
    if (e == cudaSuccess && p.do_csa)
        e = tensor_map_2d_bf16(&maps.lc, p.logit_c, p.d, rows, (uint64_t)p.d * 2, kSlice, kBoxRows, false);
    if (e == cudaSuccess && p.do_hca)
        e = tensor_map_2d_bf16(&maps.lh, p.logit_h, p.d, rows, (uint64_t)p.d * 2, kSlice, kBoxRows, false);
    if (e == cudaSuccess && p.do_csa && p.do_keys)
        e = tensor_map_2d_bf16(&maps.ki, p.idx_key, p.d_I, rows, (uint64_t)p.d_I * 2, p.d_I, kBoxRows, false);
    if (e != cudaSuccess) return e;
    int64_t span_tok = p.range_kind == 0 ? 4 * max_span : p.range_kind == 1 ? (int64_t)p.m_hca * max_span : max_span;
    const int64_t tiles = (span_tok + kTileTok - 1) / kTileTok + 1;  // the range may start inside a tile
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)tiles, (unsigned)p.B, (unsigned)(p.d / kSlice));
    if (p.norm_c || p.norm_h)  // the slices of one tile form a cluster and exchange partial sums
        return launch_kernel_cluster(compress_tile_kernel, grid, dim3(256), TileSmem::kAlloc, stream, false,
                                     dim3(1, 1, (unsigned)(p.d / kSlice)), maps, p);
    return launch_kernel(compress_tile_kernel, grid, dim3(256), TileSmem::kAlloc, stream, false, maps, p);
}

}  // namespace csa

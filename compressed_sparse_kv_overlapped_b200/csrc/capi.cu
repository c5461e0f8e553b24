// capi.cu -- the extern "C" boundary of libcsa (declared in include/csa.h): host-side argument
// validation, workspace layout, and the orchestration of the decode and prefill hot paths.
// No call allocates device memory or synchronizes the host.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>

#include "compress_dev.cuh"
#include "kernels.h"

namespace csa {

__device__ int g_status;

namespace {

thread_local std::string g_err;

// optional stage events of hybrid_attn_decode (csa_set_stage_events)
thread_local cudaEvent_t* g_events = nullptr;
thread_local int g_event_count = 0;
thread_local int g_event_cursor = 0;

cudaEvent_t next_mark() {
    if (!g_events) return nullptr;
    cudaEvent_t e = g_events[g_event_cursor];
    g_event_cursor = (g_event_cursor + 1) % g_event_count;
    return e;
}

// External records become event nodes (with timestamps) when the stream is being captured.
cudaError_t mark(cudaEvent_t e, cudaStream_t stream) {
    return e ? cudaEventRecordWithFlags(e, stream, cudaEventRecordExternal) : cudaSuccess;
}

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* where) {
    return fail(CSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

int check_dims(const csa_dims* d) {
    if (!d) return fail(CSA_ERR_ARG, "dims is NULL");
    if (d->d != 128 && d->d != 512) return fail(CSA_ERR_UNSUPPORTED, "d = %d (supported: 128, 512)", d->d);
    if (d->H < 1 || d->H > 64) return fail(CSA_ERR_UNSUPPORTED, "H = %d (supported: 1..64)", d->H);
    if (d->d_I != 32 && d->d_I != 64) return fail(CSA_ERR_UNSUPPORTED, "d_I = %d (supported: 32, 64)", d->d_I);
    if (d->d_I > d->d) return fail(CSA_ERR_UNSUPPORTED, "d_I > d");
    if (d->H_I < 1 || d->H_I > 8) return fail(CSA_ERR_UNSUPPORTED, "H_I = %d (supported: 1..8)", d->H_I);
    if (d->m != 1 && d->m != 2 && d->m != 4 && d->m != 8) return fail(CSA_ERR_UNSUPPORTED, "m = %d", d->m);
    if (d->m_hca < 1 || d->m_hca > 1024) return fail(CSA_ERR_UNSUPPORTED, "m_hca = %d", d->m_hca);
    if (d->k < 1 || d->k > kMaxK) return fail(CSA_ERR_UNSUPPORTED, "k = %d (supported: 1..%d)", d->k, kMaxK);
    if (d->W < 0 || d->W > 4096) return fail(CSA_ERR_UNSUPPORTED, "W = %d (supported: 0..4096)", d->W);
    return CSA_OK;
}

// Tuning switches from the environment, read once per process (getenv scans the whole
// environment, and the decode call sits on a per-step path).
int env_int(const char* name, int dflt) {
    static std::mutex mu;
    static const char* names[16];
    static int values[16];
    static int n = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (names[i] == name) return values[i];
    const char* v = getenv(name);
    const int r = v ? atoi(v) : dflt;
    if (n < 16) {
        names[n] = name;
        values[n] = r;
        ++n;
    }
    return r;
}

// Host checks of the optional normalization / sink parameters.
int check_norms(const csa_dims& d, const csa_norms* n) {
    if (!n) return CSA_OK;
    if (n->reserved != 0) return fail(CSA_ERR_ARG, "csa_norms.reserved must be 0");
    if (!aligned16(n->q_norm) || !aligned16(n->entry_norm_c) || !aligned16(n->entry_norm_h) ||
        (reinterpret_cast<uintptr_t>(n->sink) & 3u))
        return fail(CSA_ERR_ARG, "norm gains must be 16-byte aligned, sinks 4-byte aligned");
    if (!(n->eps >= 0.f)) return fail(CSA_ERR_ARG, "eps = %g", (double)n->eps);
    if (n->entry_norm_c && !csa_block_shape(d.m))
        return fail(CSA_ERR_UNSUPPORTED, "CSA entry normalization needs m = 4 (m = %d)", d.m);
    if (n->entry_norm_h && !hca_block_shape(d.m_hca))
        return fail(CSA_ERR_UNSUPPORTED, "HCA entry normalization needs m_hca a power of two from 4 to 128 (%d)",
                    d.m_hca);
    return CSA_OK;
}

int round64(int64_t v) { return (int)(((v + 63) / 64) * 64); }

int clamp_kpi(int64_t v, int lo, int hi) {
    int64_t r = ((v + 63) / 64) * 64;
    if (r < lo) r = lo;
    if (r > hi) r = hi;
    return (int)r;
}

// How one query's key list [front = CSA slots + window | HCA entries] is cut into attention items.
struct ItemPlan {
    int n_items, items_front, kpi_front, kpi_hca;
};

ItemPlan make_items(int64_t front_keys, int64_t max_hca, int kpi_front, int kpi_hca) {
    ItemPlan ip{};
    ip.kpi_front = kpi_front;
    ip.kpi_hca = kpi_hca;
    ip.items_front = front_keys > 0 ? (int)((front_keys + kpi_front - 1) / kpi_front) : 0;
    const int ih = max_hca > 0 ? (int)((max_hca + kpi_hca - 1) / kpi_hca) : 0;
    ip.n_items = ip.items_front + ih;
    if (ip.n_items < 1) ip.n_items = 1;  // an empty list: one empty item writing out = 0, lse = -inf
    return ip;
}

// Standalone calls: about 128 CTAs over all queries.
ItemPlan plan_standalone(int64_t front_keys, int64_t max_hca, int Q) {
    const int forced = env_int("CSA_KEYS_PER_ITEM", 0);
    const int64_t total = (front_keys + max_hca) * (int64_t)Q;
    const int kpi = forced > 0 ? round64(forced) : clamp_kpi((total + 127) / 128, 128, 2048);
    return make_items(front_keys, max_hca, kpi, kpi);
}

// SMs of the part the decode plan is sized for (B200); another count only changes the balance.
constexpr int kPlanSMs = 148;

// Decode: small front items (they run after the top-k, on the critical path); HCA items of at
// least kHcaMinKeys keys, as many as fill the SMs the front items leave free (one wave when it
// fits).  The HCA items start when the scan frees SMs and finish by the time the front items do;
// fewer, longer ones leave fewer partials to merge (measured at ctx1m: 8 tiles per item beat 5).
constexpr int kHcaMinKeys = 512;
// With CSA_DECODE_CLUSTER = 2, 4 or 8, the CTAs of each group of that many consecutive items of a
// query merge their results through distributed shared memory (one partial per group reaches the
// merge kernel); both parts' item counts are rounded up to a multiple of it (the extra items are
// empty).  Off by default: at four 1M-token sequences the rounding takes the plan from 132 CTAs to
// 160, and a cluster has to find all its SMs free in one GPC, so the items no longer fit one wave;
// the merge kernel it saves costs less than the second wave.
constexpr int kDecodeCluster = 1;
ItemPlan plan_decode_items(const csa_dims& d, int B, int64_t max_eh, int* cluster) {
    const int f = env_int("CSA_KPI_FRONT", 0), h = env_int("CSA_KPI_HCA", 0);
    const int cl = env_int("CSA_DECODE_CLUSTER", kDecodeCluster);
    *cluster = cl == 2 || cl == 4 || cl == 8 ? cl : 1;
    const int kpi_front = f > 0 ? round64(f) : 128;
    const int64_t front = (int64_t)d.k + d.W;
    const int64_t front_ctas = (int64_t)B * ((front + kpi_front - 1) / kpi_front);
    int kpi_hca;
    if (h > 0) {
        kpi_hca = round64(h);
    } else {
        const int64_t hca_ctas = front_ctas < kPlanSMs - B ? kPlanSMs - front_ctas : kPlanSMs;
        const int64_t per = ((int64_t)B * max_eh + hca_ctas - 1) / hca_ctas;
        kpi_hca = clamp_kpi(per > kHcaMinKeys ? per : kHcaMinKeys, 128, 4096);
    }
    ItemPlan ip = make_items(front, max_eh, kpi_front, kpi_hca);
    if (*cluster > 1 && ip.n_items > 1) {
        const int c = *cluster;
        const int n_hca = ip.n_items - ip.items_front;
        ip.items_front = (ip.items_front + c - 1) / c * c;
        ip.n_items = ip.items_front + (n_hca + c - 1) / c * c;
    } else {
        *cluster = 1;
    }
    return ip;
}

// ---------------------------------------------------------------------------------------------
// Decode append: one thread-block cluster of d/64 CTAs per sequence, CTA s owning channels
// [64s, 64s + 64).  len += 1 (if appending); the new token's rows (new_rows) are copied into the
// caches slice by slice; the CSA / HCA entries the token completes are compressed, each CTA its
// channel slice, with the same arithmetic as the full pass (the block-partial form of
// compress_dev.cuh where the shape allows, else the per-entry serial form); CTA 0 publishes the
// query table row; the index scratch words are cleared.  seqs[b].len is written by CTA 0 after a
// cluster barrier, once every CTA of the sequence has read the old value.
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
    grid_dep_launch();  // the scan may start its launch; it waits for this grid before reading
    __shared__ float xs[8 * 8 * 24];
    __shared__ float ss[2];  // entry normalization: this slice's sums of squares (CSA, HCA entry)
    const int s = blockIdx.x, b = blockIdx.y, ns = gridDim.x;
    const int tid = threadIdx.x;
    const csa_seq sq = p.seqs[b];
    const int64_t len = sq.len + (p.append ? 1 : 0);
    if (s == 0 && tid == 0) {
        p.queries[b].seq = b;
        p.queries[b].reserved = 0;
        p.queries[b].len = len;
    }
    if (p.zero_words) {
        const int64_t nc = (int64_t)p.B * ns, ci = (int64_t)b * ns + s;
        const int64_t per = (p.n_zero_words + nc - 1) / nc;
        const int64_t z0 = ci * per, z1 = min(p.n_zero_words, z0 + per);
        for (int64_t i = z0 + tid; i < z1; i += blockDim.x) p.zero_words[i] = 0u;
    }
    const bool ok = len >= 1;
    if (!ok && s == 0 && tid == 0) report(p.status, CSA_ERR_INDEX);
    const int d = p.d, c0s = s * 64;
    if (ok && p.append) {
        if (p.new_rows) {
            // the appended token's rows (x | logit_c | logit_h | idx_key), this CTA's channels
            const int64_t r = sq.tok_off + len - 1;
            const uint16_t* src = p.new_rows + (int64_t)b * (3 * d + p.d_I);
            const int part = tid >> 3, ch = c0s + 8 * (tid & 7);
            if (part < 3) {
                uint16_t* dst = part == 0 ? p.x : part == 1 ? p.logit_c : p.logit_h;
                *reinterpret_cast<uint4*>(dst + r * d + ch) = *reinterpret_cast<const uint4*>(src + part * d + ch);
            } else if (part == 3 && ch < p.d_I) {
                *reinterpret_cast<uint4*>(p.idx_key + r * p.d_I + ch) =
                    *reinterpret_cast<const uint4*>(src + 3 * d + ch);
            }
            __syncthreads();  // the compressor below reads these rows (coherent loads)
        }
    }
    // the entries this token completes (the same for every CTA of the sequence's cluster)
    const bool c_do = ok && p.append && len % p.m == 0;
    const bool h_do = ok && p.append && len % p.m_hca == 0;
    const int64_t j = len / p.m - 1, h = len / p.m_hca - 1;
    float cv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c_do && tid < 8) {
        const int c0 = c0s + 8 * tid;
        const int64_t row = sq.csa_off + j;
        uint4 key = make_uint4(0, 0, 0, 0);
        if (csa_block_shape(p.m)) {
            const int64_t t0 = sq.tok_off + 4 * j - 4;  // row of window position 0
            auto fetch = [&](int tensor, int pos) -> uint4 {
                const int64_t r = t0 + pos;
                if (tensor == 2) return __ldcg(reinterpret_cast<const uint4*>(p.idx_key + r * p.d_I + c0));
                const uint16_t* base = tensor == 0 ? p.logit_c : p.x;
                return __ldcg(reinterpret_cast<const uint4*>(base + r * d + c0));
            };
            if (c0 < p.d_I) {
                csa_entry_block4<true>(j, d, p.bias_c + c0, fetch, cv, &key);
                *reinterpret_cast<uint4*>(p.entry_keys + row * p.d_I + c0) = key;
            } else {
                csa_entry_block4<false>(j, d, p.bias_c + c0, fetch, cv, nullptr);
            }
        } else {  // the per-entry serial form writes the entry and its key itself (no normalization)
            compress_entry8(j, p.m, 2 * p.m, d, p.d_I, c0, p.x, p.logit_c, p.bias_c, p.idx_key, sq.tok_off,
                            p.entries + row * d, p.entry_keys + row * p.d_I);
            if (c0 < p.d_I) key = *reinterpret_cast<const uint4*>(p.entry_keys + row * p.d_I + c0);
        }
        if (p.keys_q && c0 < p.d_I) {
            // the 8-bit copy of the key (four lanes per 32-channel block)
            uint32_t sb;
            const uint2 q8 = quant_mx8(key, 0xFu << (tid & ~3), &sb);
            *reinterpret_cast<uint2*>(p.keys_q + row * p.d_I + c0) = q8;
            if ((tid & 3) == 0) p.key_scales[row * (p.d_I / 32) + c0 / 32] = (uint8_t)sb;
        }
    }
    float hv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // m' >= 16: the 16-tokens-per-warp form (warp 0 ends with the entry, two channels per lane);
    // m' = 4, 8: the 4-token block form (threads 0..7 end with it, eight channels each)
    const bool h16 = p.m_hca >= 16 && hca_block_shape(p.m_hca);
    if (h_do) {  // uniform over the CTA (both forms have barriers)
        if (h16) {
            const int w16 = tid >> 5, lane = tid & 31, wpe = p.m_hca / 16;
            const int cp = c0s + 2 * lane;
            Part2 H2;
            if (w16 < wpe) {
                const int64_t row0 = sq.tok_off + (int64_t)p.m_hca * h + 16 * w16;
                auto fetch = [&](int tensor, int t) -> uint32_t {
                    const uint16_t* base = tensor == 0 ? p.logit_h : p.x;
                    return __ldcg(reinterpret_cast<const unsigned int*>(base + (row0 + t) * d + cp));
                };
                auto bias2 = [&](int t) -> float2 {
                    return __ldg(reinterpret_cast<const float2*>(p.bias_h + (int64_t)(16 * w16 + t) * d + cp));
                };
                hca_part16(fetch, bias2, H2);
            } else {
                H2 = Part2{{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
            }
            hca_merge_warps(H2, wpe, xs);
            hv[0] = entry_div(H2.acc[0], H2.den[0]);
            hv[1] = entry_div(H2.acc[1], H2.den[1]);
        } else if (hca_block_shape(p.m_hca)) {
            const int nb = p.m_hca / 4, u = tid >> 3, g = tid & 7, ub = u & (nb - 1);
            const int c0 = c0s + 8 * g;
            const int64_t row0 = sq.tok_off + (int64_t)p.m_hca * h + 4 * ub;
            uint4 lg[4], xv[4], kv[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                lg[t] = __ldcg(reinterpret_cast<const uint4*>(p.logit_h + (row0 + t) * d + c0));
                xv[t] = __ldcg(reinterpret_cast<const uint4*>(p.x + (row0 + t) * d + c0));
                kv[t] = make_uint4(0, 0, 0, 0);
            }
            Part8 P;
            part4<false>(lg, xv, kv, p.bias_h + (int64_t)(4 * ub) * d + c0, d, P);
            hca_tree(P, nb, xs);
#pragma unroll
            for (int i = 0; i < 8; ++i) hv[i] = entry_div(P.acc[i], P.den[i]);
        } else if (tid >= 128 && tid < 136) {
            compress_entry8(h, p.m_hca, p.m_hca, d, p.d_I, c0s + 8 * (tid - 128), p.x, p.logit_h, p.bias_h,
                            nullptr, sq.tok_off, p.hca_entries + (sq.hca_off + h) * d, nullptr);
        }
    }
    float inv_c = 1.f, inv_h = 1.f;
    if ((p.norm_c || p.norm_h) && (c_do || h_do)) {
        // entry normalization (block forms only): partial sums of squares of this CTA's 64 channels,
        // then the totals over the cluster's slices, in the same order as the full pass
        if (tid < 32) {
            const float sc = sum_lane8(sumsq8(cv));
            const float sh = h16 ? warp_sum(__fmaf_rn(hv[1], hv[1], __fmaf_rn(hv[0], hv[0], 0.f)))
                                 : sum_lane8(sumsq8(hv));
            if (tid == 0) { ss[0] = sc; ss[1] = sh; }
        }
        cluster_barrier();
        if (tid < 32) {
            if (c_do && p.norm_c) inv_c = rms_inv(cluster_sum(&ss[0], ns), d, p.eps);
            if (h_do && p.norm_h) inv_h = rms_inv(cluster_sum(&ss[1], ns), d, p.eps);
        }
    }
    if (tid < 32) {
        // the entries (and their FP4 copies: threads 0..7 with eight channels each, four lanes per
        // 32-channel block)
        const int c0 = c0s + 8 * (tid & 7);
        const unsigned qmask = 0xFu << (tid & 4);
        if (c_do && csa_block_shape(p.m) && tid < 8) {
            const int64_t row = sq.csa_off + j;
            const uint4 e = entry_bf16(cv, p.norm_c ? p.norm_c + c0 : nullptr, inv_c);
            *reinterpret_cast<uint4*>(p.entries + row * d + c0) = e;
            if (p.entries_q) {
                uint32_t sb;
                *reinterpret_cast<uint32_t*>(p.entries_q + row * (d / 2) + c0 / 2) = quant_mx4(e, qmask, &sb);
                if ((tid & 3) == 0) p.entries_s[row * (d / 32) + c0 / 32] = (uint8_t)sb;
            }
        }
        if (h_do && hca_block_shape(p.m_hca)) {
            const int64_t row = sq.hca_off + h;
            uint4 e;
            if (h16) {
                const int cp = c0s + 2 * tid;
                const uint32_t hw = entry_bf16x2(hv[0], hv[1], p.norm_h ? p.norm_h + cp : nullptr, inv_h);
                *reinterpret_cast<uint32_t*>(p.hca_entries + row * d + cp) = hw;
                const int src = 4 * (tid & 7);  // the eight channels of thread t are lanes 4t .. 4t+3
                e = make_uint4(__shfl_sync(0xffffffffu, hw, src), __shfl_sync(0xffffffffu, hw, src + 1),
                               __shfl_sync(0xffffffffu, hw, src + 2), __shfl_sync(0xffffffffu, hw, src + 3));
            } else {
                e = entry_bf16(hv, p.norm_h ? p.norm_h + c0 : nullptr, inv_h);
                if (tid < 8) *reinterpret_cast<uint4*>(p.hca_entries + row * d + c0) = e;
            }
            if (p.hca_q && tid < 8) {
                uint32_t sb;
                *reinterpret_cast<uint32_t*>(p.hca_q + row * (d / 2) + c0 / 2) = quant_mx4(e, qmask, &sb);
                if ((tid & 3) == 0) p.hca_s[row * (d / 32) + c0 / 32] = (uint8_t)sb;
            }
        }
    }
    // every CTA of the sequence has read seqs[b].len: CTA 0 may now write the new length
    cluster_barrier();
    if (ok && p.append && s == 0 && tid == 0) p.seqs[b].len = len;
}

__global__ void prefill_queries_kernel(csa_query* q, int64_t p0, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        q[i].seq = 0;
        q[i].reserved = 0;
        q[i].len = p0 + i + 1;
    }
}

// ---------------------------------------------------------------------------------------------
// Workspace layouts
// ---------------------------------------------------------------------------------------------
struct DecodePlan {
    int64_t max_e;        // max CSA entries
    int64_t max_eh;       // max HCA entries
    int64_t e_stride;
    ItemPlan items;
    int cluster;          // attention items merged per thread-block cluster (1: none)
    size_t off_queries, off_idx, off_index, off_attn, total;
};

DecodePlan plan_decode(const csa_dims& d, int B, int64_t max_len) {
    DecodePlan pl{};
    pl.max_e = max_len / d.m;
    pl.max_eh = max_len / d.m_hca;
    pl.e_stride = ((pl.max_e + 3) / 4) * 4;
    if (pl.e_stride < 4) pl.e_stride = 4;
    pl.items = plan_decode_items(d, B, pl.max_eh, &pl.cluster);
    size_t off = 0;
    pl.off_queries = off;
    off += align256((size_t)B * sizeof(csa_query));
    pl.off_idx = off;
    off += align256((size_t)B * d.k * 4);
    pl.off_index = off;
    off += index_ws_bytes(B, pl.e_stride);
    pl.off_attn = off;
    off += attn_ws_bytes(B, pl.items.n_items, d.d);
    pl.total = off;
    return pl;
}

struct PrefillPlan {
    int64_t qc;           // queries per chunk
    int64_t e_stride;
    size_t off_queries, off_idx, off_index, total;
};

int sm_count(int* out);  // multiprocessors of the current device (below)

PrefillPlan plan_prefill(const csa_dims& d, int64_t q_end) {
    PrefillPlan pl{};
    const int64_t max_e = q_end / d.m;
    pl.e_stride = ((max_e + 3) / 4) * 4;
    if (pl.e_stride < 4) pl.e_stride = 4;
    // queries per chunk: by default 64 per SM, whole rounds of the persistent attention CTAs (one
    // per SM, 64 queries each, the most one holds); longer chunks also make longer score GEMMs and
    // fewer launches (measured at N = 131,072: 2,048 per chunk 56.9 ms, 4,736 = 32 x 148 53.9 ms,
    // 9,472 = 64 x 148 52.9 ms; the score rows of a chunk take 4 B x 9,472 x N/m of workspace)
    pl.qc = env_int("CSA_PREFILL_CHUNK", 0);
    if (pl.qc < 1) {
        int sms = 0;
        pl.qc = sm_count(&sms) == CSA_OK && sms > 0 ? 64 * (int64_t)sms : 9472;
    }
    size_t off = 0;
    pl.off_queries = off;
    off += align256((size_t)pl.qc * sizeof(csa_query));
    pl.off_idx = off;
    off += align256((size_t)pl.qc * d.k * 4);
    pl.off_index = off;
    off += index_ws_bytes((int)pl.qc, pl.e_stride);
    pl.total = off;
    return pl;
}

// Device address of g_status on the current device, looked up once per device (in host code the
// name g_status is a host-side stand-in, not a device address).
int status_ptr(int** out) {
    static std::mutex mu;
    static int* ptrs[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        ptrs[dev] = static_cast<int*>(p);
    }
    *out = ptrs[dev];
    return CSA_OK;
}

// Multiprocessor count of the current device, looked up once per device.
int sm_count(int* out) {
    static std::mutex mu;
    static int counts[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!counts[dev]) {
        e = cudaDeviceGetAttribute(&counts[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    }
    *out = counts[dev];
    return CSA_OK;
}

int run_index(const csa_dims& d, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_e,
              int64_t e_stride, const csa_bf16* q_idx, const float* w, const csa_bf16* entry_keys, int32_t* idx_out,
              float* score_out, void* ws_index, bool zero_ws, int* status, cudaStream_t stream,
              cudaEvent_t mid = nullptr, bool pdl = false, const void* prefetch_entries = nullptr,
              int64_t prefetch_row_bytes = 0, const uint8_t* keys_q = nullptr, const uint8_t* key_scales = nullptr,
              uint32_t* ready = nullptr) {
    IndexParams ip{};
    ip.seqs = seqs;
    ip.queries = queries;
    ip.Q = Q;
    ip.H_I = d.H_I;
    ip.d_I = d.d_I;
    ip.m = d.m;
    ip.k = d.k;
    ip.q_idx = q_idx;
    ip.w = w;
    ip.entry_keys = entry_keys;
    ip.max_entries = max_e;
    ip.idx_out = idx_out;
    ip.score_out = score_out;
    ip.status = status;
    ip.keys_q = keys_q;
    ip.key_scales = key_scales;
    ip.prefetch_rows = reinterpret_cast<const unsigned char*>(prefetch_entries);
    ip.prefetch_row_bytes = prefetch_row_bytes;
    index_ws_carve(ip, ws_index, Q, e_stride);
    ip.ready = ready;
    // with the per-step words the scan grid can select itself (when it fits the SMs): off by default.
    // At four 1M-token sequences it is slower (62.2 against 60.8 µs per step): the scan CTAs stay
    // resident through the selection, so the HCA attention items lose the SMs they otherwise take
    // while the select kernel runs on 32 of them
    if (ready && env_int("CSA_SCAN_SELECT", 0) != 0) {
        int sms = 0;
        if (sm_count(&sms) == CSA_OK) {
            ip.qsync = ready + 2 * Q;
            ip.sms = sms;
        }
    }
    if (ready) {
        uint64_t unused;
        debug_fault_state(&ip.debug_fault, &unused);
    }
    cudaError_t e = launch_index_topk(ip, max_e, stream, zero_ws, mid, pdl);
    if (e != cudaSuccess) return cuda_fail(e, "index_topk launch");
    return CSA_OK;
}

}  // namespace

int device_status(int** out) { return status_ptr(out); }

int validate_dims(const csa_dims* d) { return check_dims(d); }

namespace {
std::atomic<int> g_debug_fault{0};
std::atomic<uint64_t> g_debug_wait_ns{0};
}  // namespace

void debug_fault_state(int* fault, uint64_t* wait_ns) {
    *fault = g_debug_fault.load(std::memory_order_relaxed);
    const uint64_t w = g_debug_wait_ns.load(std::memory_order_relaxed);
    *wait_ns = w ? w : kWaitLimitNs;
}

int set_error(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

}  // namespace csa

using namespace csa;

extern "C" {

int csa_version(void) { return 200; }

int csa_debug_inject(int fault, int64_t wait_limit_ns) {
    if (fault < 0 || fault > 2)
        return fail(CSA_ERR_ARG, "fault = %d (0 none, 1 attention tile never full, 2 no ready word)", fault);
    if (wait_limit_ns < 0) return fail(CSA_ERR_ARG, "wait_limit_ns = %lld", (long long)wait_limit_ns);
    g_debug_fault.store(fault, std::memory_order_relaxed);
    g_debug_wait_ns.store((uint64_t)wait_limit_ns, std::memory_order_relaxed);
    return CSA_OK;
}

int csa_set_stage_events(void* const* events, int count) {
    if (!events || count == 0) {
        g_events = nullptr;
        g_event_count = 0;
        g_event_cursor = 0;
        return CSA_OK;
    }
    if (count < 0 || count % CSA_DECODE_MARKS) return fail(CSA_ERR_ARG, "count = %d", count);
    g_events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
    g_event_count = count;
    g_event_cursor = 0;
    return CSA_OK;
}

const char* csa_last_error(void) { return g_err.c_str(); }

int csa_sync_status(csa_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int* sp = nullptr;
    int rc = status_ptr(&sp);
    if (rc != CSA_OK) return rc;
    int v = 0;
    e = cudaMemcpy(&v, sp, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read status");
    if (v != 0) {
        int zero = 0;
        e = cudaMemcpy(sp, &zero, sizeof(int), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "clear status");
    }
    return v;
}

int csa_compress(const csa_dims* dims, int which, const csa_seq* seqs, const int64_t* ranges, int B,
                 int64_t max_entries, const csa_bf16* x, const csa_bf16* logit, const float* bias,
                 const csa_bf16* idx_key, csa_bf16* entries, csa_bf16* entry_keys, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (which != 0 && which != 1) return fail(CSA_ERR_ARG, "which = %d (0 CSA, 1 HCA)", which);
    if (!seqs || !ranges || !x || !logit || !bias || !entries) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (B < 1 || max_entries < 0) return fail(CSA_ERR_ARG, "B = %d, max_entries = %lld", B, (long long)max_entries);
    if (which == 1 && (idx_key || entry_keys)) return fail(CSA_ERR_ARG, "HCA has no indexer keys");
    if ((idx_key == nullptr) != (entry_keys == nullptr)) return fail(CSA_ERR_ARG, "idx_key and entry_keys go together");
    if (!aligned16(x) || !aligned16(logit) || !aligned16(bias) || !aligned16(entries) ||
        (idx_key && (!aligned16(idx_key) || !aligned16(entry_keys))))
        return fail(CSA_ERR_ARG, "tensors must be 16-byte aligned");
    if (max_entries == 0) return CSA_OK;
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    cudaError_t e;
    if (which == 0 ? csa_block_shape(dims->m) : hca_block_shape(dims->m_hca)) {
        TileCompressParams tp{};
        tp.seqs = seqs;
        tp.ranges = ranges;
        tp.range_kind = which;
        tp.B = B;
        tp.d = dims->d;
        tp.d_I = dims->d_I;
        tp.m_hca = dims->m_hca;
        tp.do_csa = which == 0;
        tp.do_hca = which == 1;
        tp.do_keys = idx_key != nullptr;
        tp.x = x;
        tp.logit_c = which == 0 ? logit : nullptr;
        tp.logit_h = which == 1 ? logit : nullptr;
        tp.idx_key = idx_key;
        tp.bias_c = which == 0 ? bias : nullptr;
        tp.bias_h = which == 1 ? bias : nullptr;
        tp.entries = which == 0 ? entries : nullptr;
        tp.entry_keys = entry_keys;
        tp.hca_entries = which == 1 ? entries : nullptr;
        tp.status = st;
        e = launch_compress_tiles(tp, max_entries, stream);
    } else {
        CompressParams p{};
        p.seqs = seqs;
        p.ranges = ranges;
        p.B = B;
        p.which = which;
        p.d = dims->d;
        p.d_I = dims->d_I;
        p.m = which ? dims->m_hca : dims->m;
        p.win = which ? dims->m_hca : 2 * dims->m;
        p.x = x;
        p.logit = logit;
        p.bias = bias;
        p.idx_key = idx_key;
        p.entries = entries;
        p.entry_keys = entry_keys;
        p.status = st;
        e = launch_compress(p, max_entries, stream);
    }
    return e == cudaSuccess ? CSA_OK : cuda_fail(e, "compress launch");
}

// Both caches for token ranges (one pass over the raw rows when both ratios have the block form).
static int compress_all(const csa_dims& d, const csa_seq* seqs, const int64_t* tok_ranges, int64_t t0, int64_t t1,
                        int B, int64_t max_tokens, const csa_bf16* x, const csa_bf16* logit_c,
                        const csa_bf16* logit_h, const float* bias_c, const float* bias_h, const csa_bf16* idx_key,
                        csa_bf16* entries, csa_bf16* entry_keys, csa_bf16* hca_entries, const csa_norms* norms,
                        int* st, cudaStream_t stream) {
    const bool csa_blk = csa_block_shape(d.m), hca_blk = hca_block_shape(d.m_hca);
    TileCompressParams tp{};
    tp.seqs = seqs;
    tp.ranges = tok_ranges;
    tp.range_begin = t0;
    tp.range_end = t1;
    tp.range_kind = 2;
    tp.B = B;
    tp.d = d.d;
    tp.d_I = d.d_I;
    tp.m_hca = d.m_hca;
    tp.do_csa = csa_blk;
    tp.do_hca = hca_blk;
    tp.do_keys = 1;
    tp.x = x;
    tp.logit_c = logit_c;
    tp.logit_h = logit_h;
    tp.idx_key = idx_key;
    tp.bias_c = bias_c;
    tp.bias_h = bias_h;
    tp.entries = entries;
    tp.entry_keys = entry_keys;
    tp.hca_entries = hca_entries;
    if (norms) {
        tp.norm_c = norms->entry_norm_c;
        tp.norm_h = norms->entry_norm_h;
        tp.eps = norms->eps;
    }
    tp.status = st;
    cudaError_t e = launch_compress_tiles(tp, max_tokens, stream);
    if (e != cudaSuccess) return cuda_fail(e, "compress launch");
    for (int which = 0; which < 2; ++which) {
        if (which == 0 ? csa_blk : hca_blk) continue;
        const int m = which ? d.m_hca : d.m;
        if (max_tokens / m + 1 <= 0) continue;
        CompressParams p{};
        p.seqs = seqs;
        p.ranges = tok_ranges;
        p.range_begin = t0;
        p.range_end = t1;
        p.token_ranges = 1;
        p.B = B;
        p.which = which;
        p.d = d.d;
        p.d_I = d.d_I;
        p.m = m;
        p.win = which ? d.m_hca : 2 * d.m;
        p.x = x;
        p.logit = which ? logit_h : logit_c;
        p.bias = which ? bias_h : bias_c;
        p.idx_key = which ? nullptr : idx_key;
        p.entries = which ? hca_entries : entries;
        p.entry_keys = which ? nullptr : entry_keys;
        p.status = st;
        if ((e = launch_compress(p, max_tokens / m + 1, stream)) != cudaSuccess) return cuda_fail(e, "compress launch");
    }
    return CSA_OK;
}

int csa_compress_all(const csa_dims* dims, const csa_seq* seqs, const int64_t* tok_ranges, int B, int64_t max_tokens,
                     const csa_bf16* x, const csa_bf16* logit_c, const csa_bf16* logit_h, const float* bias_c,
                     const float* bias_h, const csa_bf16* idx_key, csa_bf16* entries, csa_bf16* entry_keys,
                     csa_bf16* hca_entries, const csa_norms* norms, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_norms(*dims, norms))) return rc;
    if (!seqs || !tok_ranges || !x || !logit_c || !logit_h || !bias_c || !bias_h || !idx_key || !entries ||
        !entry_keys || !hca_entries)
        return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (B < 1 || max_tokens < 0) return fail(CSA_ERR_ARG, "B = %d, max_tokens = %lld", B, (long long)max_tokens);
    if (!aligned16(x) || !aligned16(logit_c) || !aligned16(logit_h) || !aligned16(bias_c) || !aligned16(bias_h) ||
        !aligned16(idx_key) || !aligned16(entries) || !aligned16(entry_keys) || !aligned16(hca_entries))
        return fail(CSA_ERR_ARG, "tensors must be 16-byte aligned");
    if (max_tokens == 0) return CSA_OK;
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    return compress_all(*dims, seqs, tok_ranges, 0, 0, B, max_tokens, x, logit_c, logit_h, bias_c, bias_h, idx_key,
                        entries, entry_keys, hca_entries, norms, st, stream);
}

size_t csa_workspace_size(int op, const void* args) {
    if (!args) return 0;
    if (op == CSA_OP_INDEX_TOPK || op == CSA_OP_SPARSE_ATTN || op == CSA_OP_HCA_ATTN) {
        const csa_ws_query* a = static_cast<const csa_ws_query*>(args);
        if (check_dims(&a->dims) || a->Q < 1 || a->max_len < 0) return 0;
        if (op == CSA_OP_INDEX_TOPK) {
            int64_t es = ((a->max_len / a->dims.m + 3) / 4) * 4;
            if (es < 4) es = 4;
            return index_ws_bytes(a->Q, es) + 256;
        }
        const ItemPlan ip = op == CSA_OP_SPARSE_ATTN
                                ? plan_standalone((int64_t)a->dims.k + a->dims.W, 0, a->Q)
                                : plan_standalone(a->dims.W, a->max_len / a->dims.m_hca, a->Q);
        return attn_ws_bytes(a->Q, ip.n_items, a->dims.d) + 256;
    }
    if (op == CSA_OP_DECODE) {
        const csa_decode_args* a = static_cast<const csa_decode_args*>(args);
        if (check_dims(&a->dims) || a->B < 1 || a->max_len < 1) return 0;
        return plan_decode(a->dims, a->B, a->max_len).total;
    }
    if (op == CSA_OP_PREFILL) {
        const csa_prefill_args* a = static_cast<const csa_prefill_args*>(args);
        if (check_dims(&a->dims) || a->q_end < 1) return 0;
        return plan_prefill(a->dims, a->q_end).total;
    }
    return 0;
}

int csa_index_topk(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                   const csa_bf16* q_idx, const float* w, const csa_bf16* entry_keys, int32_t* idx_out,
                   float* score_out, void* ws, size_t ws_bytes, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q_idx || !w || !entry_keys || !idx_out) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (Q < 1 || max_len < 1) return fail(CSA_ERR_ARG, "Q = %d, max_len = %lld", Q, (long long)max_len);
    if (!aligned16(q_idx) || !aligned16(entry_keys)) return fail(CSA_ERR_ARG, "q_idx / entry_keys must be 16-byte aligned");
    csa_ws_query wq{*dims, Q, 0, max_len};
    const size_t need = csa_workspace_size(CSA_OP_INDEX_TOPK, &wq);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", need);
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    const int64_t max_e = max_len / dims->m;
    int64_t es = ((max_e + 3) / 4) * 4;
    if (es < 4) es = 4;
    return run_index(*dims, seqs, queries, Q, max_e, es, q_idx, w, entry_keys, idx_out, score_out, ws, true, st,
                     stream);
}

int csa_quantize_keys(const csa_dims* dims, const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries,
                      const csa_bf16* entry_keys, uint8_t* keys_q, uint8_t* key_scales, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !ranges || !entry_keys || !keys_q || !key_scales) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (B < 1 || max_entries < 0) return fail(CSA_ERR_ARG, "B = %d, max_entries = %lld", B, (long long)max_entries);
    if (!aligned16(entry_keys) || !aligned16(keys_q)) return fail(CSA_ERR_ARG, "entry_keys / keys_q must be 16-byte aligned");
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    cudaError_t e = launch_quantize_keys(seqs, ranges, B, max_entries, dims->m, dims->d_I, entry_keys, keys_q,
                                         key_scales, st, stream);
    return e == cudaSuccess ? CSA_OK : cuda_fail(e, "quantize launch");
}

int csa_index_topk_mx8(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                       const csa_bf16* q_idx, const float* w, const uint8_t* keys_q, const uint8_t* key_scales,
                       int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q_idx || !w || !keys_q || !key_scales || !idx_out)
        return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (Q < 1 || max_len < 1) return fail(CSA_ERR_ARG, "Q = %d, max_len = %lld", Q, (long long)max_len);
    if (!aligned16(q_idx) || !aligned16(keys_q) || (reinterpret_cast<uintptr_t>(key_scales) & 1u))
        return fail(CSA_ERR_ARG, "q_idx / keys_q must be 16-byte aligned, key_scales 2-byte aligned");
    csa_ws_query wq{*dims, Q, 0, max_len};
    const size_t need = csa_workspace_size(CSA_OP_INDEX_TOPK, &wq);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", need);
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    const int64_t max_e = max_len / dims->m;
    int64_t es = ((max_e + 3) / 4) * 4;
    if (es < 4) es = 4;
    return run_index(*dims, seqs, queries, Q, max_e, es, q_idx, w, nullptr, idx_out, score_out, ws, true, st, stream,
                     nullptr, false, nullptr, 0, keys_q, key_scales);
}

// FP4 entry caches (codes and block scales) an attention call reads instead of the bf16 ones.
struct Fp4Caches {
    const uint8_t* entries_q = nullptr;
    const uint8_t* entries_s = nullptr;
    const uint8_t* hca_q = nullptr;
    const uint8_t* hca_s = nullptr;
};

static int make_attn(AttnParams& p, const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q,
                     const csa_bf16* q, const csa_bf16* entries, const int32_t* idx, int k_slots, const csa_bf16* x,
                     int W, const csa_bf16* hca, float scale, float* out, float* lse, void* ws, const ItemPlan& ip,
                     const csa_norms* norms = nullptr, const Fp4Caches& fp4 = Fp4Caches{}) {
    int* st = nullptr;
    int rc = status_ptr(&st);
    if (rc) return rc;
    if (ip.n_items < 1 || ip.n_items > 256)
        return fail(CSA_ERR_UNSUPPORTED, "%d attention items per query (1..256)", ip.n_items);
    p = AttnParams{};
    p.seqs = seqs;
    p.queries = queries;
    p.Q = Q;
    p.H = dims->H;
    p.d = dims->d;
    p.q = q;
    p.entries = entries;
    p.idx = idx;
    p.k_slots = k_slots;
    p.m = dims->m;
    p.raw = x;
    p.W = W;
    p.hca = hca;
    p.entries_q = fp4.entries_q;
    p.entries_s = fp4.entries_s;
    p.hca_q = fp4.hca_q;
    p.hca_s = fp4.hca_s;
    p.m_hca = dims->m_hca;
    p.use_hca = hca != nullptr || fp4.hca_q != nullptr;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_items = ip.n_items;
    p.items_front = ip.items_front;
    p.kpi_front = ip.kpi_front;
    p.kpi_hca = ip.kpi_hca;
    p.out = out;
    p.lse = lse;
    if (norms) {
        p.sink = norms->sink;
        p.q_norm = norms->q_norm;
        p.norm_eps = norms->eps;
    }
    p.status = st;
    debug_fault_state(&p.debug_fault, &p.wait_ns);
    p.persist = env_int("CSA_ATTN_PERSIST", 1) != 0;
    attn_ws_carve(p, ws);
    return CSA_OK;
}

static int run_attention_all(const AttnParams& p, cudaStream_t stream) {
    cudaError_t e = launch_attention_items(p, 0, p.n_items, stream);
    if (e == cudaSuccess) e = launch_combine(p, stream);
    return e == cudaSuccess ? CSA_OK : cuda_fail(e, "attention launch");
}

int csa_sparse_attn(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, const csa_bf16* q,
                    const csa_bf16* entries, const int32_t* idx, const csa_bf16* x, float scale, float* out,
                    float* lse, void* ws, size_t ws_bytes, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q || !entries || !idx || !x || !out) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (Q < 1) return fail(CSA_ERR_ARG, "Q = %d", Q);
    if (!aligned16(q) || !aligned16(entries) || !aligned16(x) || !aligned16(out))
        return fail(CSA_ERR_ARG, "q / entries / x / out must be 16-byte aligned");
    csa_ws_query wq{*dims, Q, 0, 1};
    const size_t need = csa_workspace_size(CSA_OP_SPARSE_ATTN, &wq);
    if (need > 256 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", need);
    AttnParams p;
    int rc2 = make_attn(p, dims, seqs, queries, Q, q, entries, idx, dims->k, x, dims->W, nullptr, scale, out, lse, ws,
                        plan_standalone((int64_t)dims->k + dims->W, 0, Q));
    if (rc2) return rc2;
    return run_attention_all(p, stream);
}

int hca_dense_attn(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                   const csa_bf16* q, const csa_bf16* hca_entries, const csa_bf16* x, int W, float scale, float* out,
                   float* lse, void* ws, size_t ws_bytes, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q || !hca_entries || !x || !out) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (Q < 1 || max_len < 1 || W < 0 || W > 4096) return fail(CSA_ERR_ARG, "Q = %d, max_len, W = %d", Q, W);
    if (!aligned16(q) || !aligned16(hca_entries) || !aligned16(x) || !aligned16(out))
        return fail(CSA_ERR_ARG, "q / hca_entries / x / out must be 16-byte aligned");
    csa_dims d2 = *dims;
    d2.W = W;
    csa_ws_query wq{d2, Q, 0, max_len};
    const size_t need = csa_workspace_size(CSA_OP_HCA_ATTN, &wq);
    if (need > 256 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", need);
    // key list: [raw window | HCA entries] (no CSA slots)
    AttnParams p;
    int rc2 = make_attn(p, &d2, seqs, queries, Q, q, nullptr, nullptr, 0, x, W, hca_entries, scale, out, lse, ws,
                        plan_standalone(W, max_len / dims->m_hca, Q));
    if (rc2) return rc2;
    return run_attention_all(p, stream);
}

int csa_quantize_entries(const csa_dims* dims, const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries,
                         int which, const csa_bf16* entries, uint8_t* entries_q, uint8_t* entry_scales,
                         csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !ranges || !entries || !entries_q || !entry_scales) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (which != 0 && which != 1) return fail(CSA_ERR_ARG, "which = %d (0 CSA, 1 HCA)", which);
    if (B < 1 || max_entries < 0) return fail(CSA_ERR_ARG, "B = %d, max_entries = %lld", B, (long long)max_entries);
    if (!aligned16(entries) || !aligned16(entries_q)) return fail(CSA_ERR_ARG, "entries / entries_q must be 16-byte aligned");
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    cudaError_t e = launch_quantize_entries(seqs, ranges, B, max_entries, which, which ? dims->m_hca : dims->m,
                                            dims->d, entries, entries_q, entry_scales, st, stream);
    return e == cudaSuccess ? CSA_OK : cuda_fail(e, "quantize launch");
}

int csa_sparse_attn_fp4(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, const csa_bf16* q,
                        const uint8_t* entries_q, const uint8_t* entry_scales, const int32_t* idx, const csa_bf16* x,
                        float scale, float* out, float* lse, void* ws, size_t ws_bytes, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q || !entries_q || !entry_scales || !idx || !x || !out)
        return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (Q < 1) return fail(CSA_ERR_ARG, "Q = %d", Q);
    if (!aligned16(q) || !aligned16(entries_q) || !aligned16(x) || !aligned16(out))
        return fail(CSA_ERR_ARG, "q / entries_q / x / out must be 16-byte aligned");
    csa_ws_query wq{*dims, Q, 0, 1};
    const size_t need = csa_workspace_size(CSA_OP_SPARSE_ATTN, &wq);
    if (need > 256 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", need);
    Fp4Caches f4;
    f4.entries_q = entries_q;
    f4.entries_s = entry_scales;
    AttnParams p;
    int rc2 = make_attn(p, dims, seqs, queries, Q, q, nullptr, idx, dims->k, x, dims->W, nullptr, scale, out, lse, ws,
                        plan_standalone((int64_t)dims->k + dims->W, 0, Q), nullptr, f4);
    if (rc2) return rc2;
    return run_attention_all(p, stream);
}

int hca_dense_attn_fp4(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                       const csa_bf16* q, const uint8_t* hca_q, const uint8_t* hca_scales, const csa_bf16* x, int W,
                       float scale, float* out, float* lse, void* ws, size_t ws_bytes, csa_stream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!seqs || !queries || !q || !hca_q || !hca_scales || !x || !out) return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (Q < 1 || max_len < 1 || W < 0 || W > 4096) return fail(CSA_ERR_ARG, "Q = %d, max_len, W = %d", Q, W);
    if (!aligned16(q) || !aligned16(hca_q) || !aligned16(x) || !aligned16(out))
        return fail(CSA_ERR_ARG, "q / hca_q / x / out must be 16-byte aligned");
    csa_dims d2 = *dims;
    d2.W = W;
    csa_ws_query wq{d2, Q, 0, max_len};
    const size_t need = csa_workspace_size(CSA_OP_HCA_ATTN, &wq);
    if (need > 256 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", need);
    Fp4Caches f4;
    f4.hca_q = hca_q;
    f4.hca_s = hca_scales;
    AttnParams p;
    int rc2 = make_attn(p, &d2, seqs, queries, Q, q, nullptr, nullptr, 0, x, W, nullptr, scale, out, lse, ws,
                        plan_standalone(W, max_len / dims->m_hca, Q), nullptr, f4);
    if (rc2) return rc2;
    return run_attention_all(p, stream);
}

int hybrid_attn_decode(const csa_decode_args* a, void* ws, size_t ws_bytes, csa_stream_t stream) {
    if (!a) return fail(CSA_ERR_ARG, "args is NULL");
    int rc = check_dims(&a->dims);
    if (rc) return rc;
    const csa_dims& d = a->dims;
    if (a->B < 1 || a->max_len < 1) return fail(CSA_ERR_ARG, "B = %d, max_len = %lld", a->B, (long long)a->max_len);
    // with idx_in (a selection reused from another layer) the indexer does not run: no indexer query
    const bool reuse = a->idx_in != nullptr;
    if (!a->seqs || !a->x || !a->logit_c || !a->logit_h || !a->idx_key || !a->bias_c || !a->bias_h || !a->entries ||
        !a->entry_keys || !a->hca_entries || !a->q || (!reuse && (!a->q_idx || !a->w)) || !a->out)
        return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (!aligned16(a->x) || !aligned16(a->logit_c) || !aligned16(a->logit_h) || !aligned16(a->idx_key) ||
        !aligned16(a->bias_c) || !aligned16(a->bias_h) || !aligned16(a->entries) || !aligned16(a->entry_keys) ||
        !aligned16(a->hca_entries) || !aligned16(a->q) || !aligned16(a->q_idx) || !aligned16(a->out) ||
        !aligned16(a->new_rows))
        return fail(CSA_ERR_ARG, "tensors must be 16-byte aligned");
    if (reuse && a->idx_out) return fail(CSA_ERR_ARG, "idx_out with idx_in (the selection is the caller's)");
    if ((rc = check_norms(d, a->norms))) return rc;
    if (a->new_rows && !a->append) return fail(CSA_ERR_ARG, "new_rows without append");
    if ((a->keys_q == nullptr) != (a->key_scales == nullptr)) return fail(CSA_ERR_ARG, "keys_q and key_scales go together");
    const bool fp4 = a->entries_q != nullptr;
    if (fp4 != (a->entry_scales != nullptr) || fp4 != (a->hca_q != nullptr) || fp4 != (a->hca_scales != nullptr))
        return fail(CSA_ERR_ARG, "entries_q, entry_scales, hca_q and hca_scales go together");
    if (fp4 && (!aligned16(a->entries_q) || !aligned16(a->hca_q)))
        return fail(CSA_ERR_ARG, "entries_q / hca_q must be 16-byte aligned");
    if (fp4 && (!csa_block_shape(d.m) || !hca_block_shape(d.m_hca)))
        return fail(CSA_ERR_UNSUPPORTED, "FP4 entry caches need m = 4 and m_hca a power of two from 4 to 128");
    if (a->keys_q && (!aligned16(a->keys_q) || (reinterpret_cast<uintptr_t>(a->key_scales) & 1u)))
        return fail(CSA_ERR_ARG, "keys_q must be 16-byte aligned, key_scales 2-byte aligned");
    const DecodePlan pl = plan_decode(d, a->B, a->max_len);
    if (!ws || ws_bytes < pl.total || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", pl.total);
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    char* w = static_cast<char*>(ws);
    csa_query* queries = reinterpret_cast<csa_query*>(w + pl.off_queries);
    int32_t* idx = reuse ? const_cast<int32_t*>(a->idx_in)
                         : a->idx_out ? a->idx_out : reinterpret_cast<int32_t*>(w + pl.off_idx);
    void* ws_index = w + pl.off_index;

    AppendParams ap{};
    ap.seqs = a->seqs;
    ap.B = a->B;
    ap.append = a->append ? 1 : 0;
    ap.d = d.d;
    ap.d_I = d.d_I;
    ap.m = d.m;
    ap.m_hca = d.m_hca;
    ap.x = a->x;
    ap.logit_c = a->logit_c;
    ap.logit_h = a->logit_h;
    ap.idx_key = a->idx_key;
    ap.new_rows = a->new_rows;
    ap.bias_c = a->bias_c;
    ap.bias_h = a->bias_h;
    ap.entries = a->entries;
    ap.entry_keys = a->entry_keys;
    ap.hca_entries = a->hca_entries;
    ap.keys_q = a->keys_q;
    ap.key_scales = a->key_scales;
    ap.entries_q = a->entries_q;
    ap.entries_s = a->entry_scales;
    ap.hca_q = a->hca_q;
    ap.hca_s = a->hca_scales;
    if (a->norms) {
        ap.norm_c = a->norms->entry_norm_c;
        ap.norm_h = a->norms->entry_norm_h;
        ap.eps = a->norms->eps;
    }
    ap.queries = queries;
    ap.zero_words = static_cast<uint32_t*>(ws_index);  // histograms + ready words of the index scratch
    ap.n_zero_words = (int64_t)(index_zero_bytes(a->B) / 4);
    ap.status = st;
    cudaEvent_t ev[CSA_DECODE_MARKS] = {};
    for (int i = 0; i < CSA_DECODE_MARKS; ++i) ev[i] = next_mark();
    cudaError_t e = mark(ev[0], stream);
    if (e == cudaSuccess) e = launch_append(ap, stream);
    if (e == cudaSuccess) e = mark(ev[1], stream);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    AttnParams ap2;
    Fp4Caches f4;
    f4.entries_q = a->entries_q;
    f4.entries_s = a->entry_scales;
    f4.hca_q = a->hca_q;
    f4.hca_s = a->hca_scales;
    rc = make_attn(ap2, &d, a->seqs, queries, a->B, a->q, a->entries, idx, d.k, a->x, d.W, a->hca_entries, a->scale,
                   a->out, a->lse, w + pl.off_attn, pl.items, a->norms, f4);
    if (rc) return rc;
    // programmatic dependent launch chains append -> scan -> select -> attention -> merge unless
    // stage events are being recorded between them
    const bool pdl = ev[0] == nullptr && env_int("CSA_NO_PDL", 0) == 0;
    // every item in one launch after the top-k; the HCA items need no top-k and start as soon as the
    // scan frees SMs (their inputs, written by the append, are two launches back; with a reused
    // selection the append is the launch right before, so they wait like the others)
    ap2.hca_nowait = (pdl && !reuse) ? 1 : 0;
    ap2.queries_early = reuse ? 0 : 1;  // the append is two launches back only with the indexer between
    ap2.hca_first = (pl.items.n_items > 1 && pl.items.items_front > 0) ? 1 : 0;
    ap2.cluster = pl.cluster;
    // per-step words cleared by the append: the front items start on their query's ready word from
    // the select, and the merge of a query on its item counter, not on the end of the previous grid
    uint32_t* step_words = index_ready_words(ws_index, a->B);
    uint32_t* ready = reuse ? nullptr : step_words;
    ap2.ready = pl.items.n_items > 1 ? ready : nullptr;
    ap2.items_done = pl.items.n_items > 1 ? step_words + a->B : nullptr;
    if (!reuse) {
        rc = run_index(d, a->seqs, queries, a->B, pl.max_e, pl.e_stride, a->q_idx, a->w, a->entry_keys, idx, nullptr,
                       ws_index, false, st, stream, ev[2], pdl,
                       fp4 ? static_cast<const void*>(a->entries_q) : static_cast<const void*>(a->entries),
                       fp4 ? (int64_t)d.d / 2 : (int64_t)d.d * 2, a->keys_q, a->key_scales, ready);
        if (rc) return rc;
    } else if ((e = mark(ev[2], stream)) != cudaSuccess) {
        return cuda_fail(e, "event record");
    }
    if ((e = mark(ev[3], stream)) != cudaSuccess) return cuda_fail(e, "event record");
    e = launch_attention_items(ap2, 0, pl.items.n_items, stream, pdl);
    if (e == cudaSuccess) e = launch_combine(ap2, stream, pdl);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    if ((e = mark(ev[4], stream)) != cudaSuccess) return cuda_fail(e, "event record");
    return CSA_OK;
}

int hybrid_attn_prefill(const csa_prefill_args* a, void* ws, size_t ws_bytes, csa_stream_t stream) {
    if (!a) return fail(CSA_ERR_ARG, "args is NULL");
    int rc = check_dims(&a->dims);
    if (rc) return rc;
    const csa_dims& d = a->dims;
    if (a->q_begin < 0 || a->q_end <= a->q_begin || a->q_end > a->len)
        return fail(CSA_ERR_ARG, "query range [%lld, %lld) of len %lld", (long long)a->q_begin, (long long)a->q_end,
                    (long long)a->len);
    const bool reuse = a->idx_in != nullptr;  // a selection reused from another layer: no indexer
    if (!a->seq || !a->x || !a->logit_c || !a->logit_h || !a->idx_key || !a->bias_c || !a->bias_h || !a->entries ||
        !a->entry_keys || !a->hca_entries || !a->q || (!reuse && (!a->q_idx || !a->w)) || !a->out)
        return fail(CSA_ERR_ARG, "NULL pointer argument");
    if (!aligned16(a->x) || !aligned16(a->logit_c) || !aligned16(a->logit_h) || !aligned16(a->idx_key) ||
        !aligned16(a->bias_c) || !aligned16(a->bias_h) || !aligned16(a->entries) || !aligned16(a->entry_keys) ||
        !aligned16(a->hca_entries) || !aligned16(a->q) || !aligned16(a->q_idx) || !aligned16(a->out))
        return fail(CSA_ERR_ARG, "tensors must be 16-byte aligned");
    if (reuse && a->idx_out) return fail(CSA_ERR_ARG, "idx_out with idx_in (the selection is the caller's)");
    if ((rc = check_norms(d, a->norms))) return rc;
    const PrefillPlan pl = plan_prefill(d, a->q_end);
    if (!ws || ws_bytes < pl.total || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(CSA_ERR_ARG, "workspace: need %zu bytes, 256-byte aligned", pl.total);
    int* st = nullptr;
    if ((rc = status_ptr(&st))) return rc;
    cudaError_t e;
    if (a->compress) {
        // every CSA and HCA entry complete in [0, q_end): one pass over the raw rows
        rc = compress_all(d, a->seq, nullptr, 0, a->q_end, 1, a->q_end, a->x, a->logit_c, a->logit_h, a->bias_c,
                          a->bias_h, a->idx_key, a->entries, a->entry_keys, a->hca_entries, a->norms, st, stream);
        if (rc) return rc;
    }
    char* w = static_cast<char*>(ws);
    csa_query* queries = reinterpret_cast<csa_query*>(w + pl.off_queries);
    // the indexer runs as a tensor-core GEMM when its shape allows (d_I = 64, H_I <= 4, rows that fit
    // the select's shared memory); CSA_PREFILL_SCAN=1 forces the per-query scan
    const bool gemm_index = d.d_I == 64 && d.H_I <= 4 && a->q_end / d.m <= kSelRowMax &&
                            env_int("CSA_PREFILL_SCAN", 0) == 0;
    for (int64_t p0 = a->q_begin; p0 < a->q_end; p0 += pl.qc) {
        const int64_t n = a->q_end - p0 < pl.qc ? a->q_end - p0 : pl.qc;
        const int64_t r0 = p0 - a->q_begin;
        if ((e = launch_prefill_queries(queries, p0, n, stream)) != cudaSuccess) return cuda_fail(e, "query table");
        int32_t* idx = reuse ? const_cast<int32_t*>(a->idx_in) + r0 * d.k
                             : a->idx_out ? a->idx_out + r0 * d.k : reinterpret_cast<int32_t*>(w + pl.off_idx);
        // the chunk's queries see at most p0 + n tokens: size the indexer for that, not for q_end
        const int64_t max_e_chunk = (p0 + n) / d.m;
        if (reuse) {
            // the selection is the source layer's
        } else if (gemm_index) {
            // scores of the whole chunk as one tensor-core GEMM, then a sampled-threshold select
            IndexParams ip{};
            ip.seqs = a->seq;
            ip.queries = queries;
            ip.Q = (int)n;
            ip.H_I = d.H_I;
            ip.d_I = d.d_I;
            ip.m = d.m;
            ip.k = d.k;
            ip.q_idx = a->q_idx + r0 * d.H_I * d.d_I;
            ip.w = a->w + r0 * d.H_I;
            ip.entry_keys = a->entry_keys;
            ip.max_entries = max_e_chunk;
            ip.idx_out = idx;
            ip.score_out = nullptr;
            ip.status = st;
            index_ws_carve(ip, w + pl.off_index, (int)n, pl.e_stride);
            if (max_e_chunk > d.k) {
                PrefillScoreParams sp{};
                sp.seq = a->seq;
                sp.q_idx = ip.q_idx;
                sp.w = ip.w;
                sp.entry_keys = a->entry_keys;
                sp.H_I = d.H_I;
                sp.m_shift = d.m == 1 ? 0 : d.m == 2 ? 1 : d.m == 4 ? 2 : 3;  // m is 1, 2, 4 or 8
                sp.Qn = (int)n;
                sp.pos0 = p0;
                // entry ranges for two waves of one CTA per SM: at most 2 x SMs CTAs in all (ranges
                // rounded up to whole tiles, so that a few leftover CTAs never form a third wave)
                const int64_t gy = (n + 127) / 128;
                int sms = 148;
                if (sm_count(&sms) != CSA_OK) sms = 148;
                const int64_t gx_max = 2 * (int64_t)sms / gy > 0 ? 2 * (int64_t)sms / gy : 1;
                int64_t ent = (max_e_chunk + gx_max - 1) / gx_max;
                ent = ((ent + 63) / 64) * 64;
                sp.ent_per_cta = ent < 64 ? 64 : ent;
                sp.scores = ip.scores;
                sp.e_stride = ip.e_stride;
                sp.status = st;
                if ((e = launch_prefill_scores(sp, max_e_chunk, stream)) != cudaSuccess)
                    return cuda_fail(e, "prefill score launch");
            }
            if ((e = launch_index_topk(ip, max_e_chunk, stream, false, nullptr, false, true)) != cudaSuccess)
                return cuda_fail(e, "select launch");
        } else {
            rc = run_index(d, a->seq, queries, (int)n, max_e_chunk, pl.e_stride, a->q_idx + r0 * d.H_I * d.d_I,
                           a->w + r0 * d.H_I, a->entry_keys, idx, nullptr, w + pl.off_index, true, st, stream);
            if (rc) return rc;
        }
        AttnParams pp;
        ItemPlan one{1, 0, 64, 64};
        rc = make_attn(pp, &d, a->seq, queries, (int)n, a->q + r0 * d.H * d.d, a->entries, idx, d.k, a->x, d.W,
                       a->hca_entries, a->scale, a->out + r0 * d.H * d.d, a->lse ? a->lse + r0 * d.H : nullptr, nullptr,
                       one, a->norms);
        if (rc) return rc;
        if ((rc = run_attention_all(pp, stream))) return rc;
    }
    return CSA_OK;
}

}  // extern "C"

namespace csa {

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
    const unsigned ns = (unsigned)(p.d / 64);
    return launch_kernel_cluster(append_kernel, dim3(ns, (unsigned)p.B), dim3(256), 0, stream, false, dim3(ns, 1, 1), p);
}

cudaError_t launch_prefill_queries(csa_query* queries, int64_t p0, int64_t n, cudaStream_t stream) {
    int64_t blocks = (n + 255) / 256;
    if (blocks > 1024) blocks = 1024;
    prefill_queries_kernel<<<(unsigned)blocks, 256, 0, stream>>>(queries, p0, n);
    return cudaGetLastError();
}

}  // namespace csa

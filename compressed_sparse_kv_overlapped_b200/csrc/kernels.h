// kernels.h -- internal launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

struct CompressParams {
    const csa_seq* seqs;
    const int64_t* ranges;   // [B][2], or nullptr: every sequence uses [range_begin, range_end)
    int64_t range_begin, range_end;
    int token_ranges;        // 1: the ranges are token ranges [t0, t1): entries [t0/m, t1/m)
    int B;
    int which;               // 0 CSA, 1 HCA
    int d, d_I, m, win;
    const uint16_t* x;
    const uint16_t* logit;
    const float* bias;
    const uint16_t* idx_key; // nullable
    uint16_t* entries;
    uint16_t* entry_keys;    // nullable
    int* status;
};
cudaError_t launch_compress(const CompressParams& p, int64_t max_entries, cudaStream_t stream);

// Block-partial compressor (compress_dev.cuh) over 128-token tiles staged by TMA: one CTA per
// (tile, sequence, 64-channel slice) computes the tile's CSA entries (with indexer keys) and HCA
// entries from one read of each token row.  Shapes: CSA ratio 4; HCA ratio a power of two from 4 to
// 128; d a multiple of 64; d_I 32 or 64.  The decode append uses the same arithmetic for the same
// shapes, so both produce identical entries.
__host__ __device__ constexpr bool csa_block_shape(int m) { return m == 4; }  // CSA by the block-partial form
__host__ __device__ constexpr bool hca_block_shape(int m_hca) {             // HCA by the block-partial form
    return m_hca >= 4 && m_hca <= 128 && (m_hca & (m_hca - 1)) == 0;
}
struct TileCompressParams {
    const csa_seq* seqs;
    const int64_t* ranges;    // [B][2] or nullptr: every sequence uses [range_begin, range_end)
    int64_t range_begin, range_end;
    int range_kind;           // 0: CSA entry range, 1: HCA entry range, 2: token range (both caches)
    int B, d, d_I, m_hca;
    int do_csa, do_hca, do_keys;
    const uint16_t* x;
    const uint16_t* logit_c;
    const uint16_t* logit_h;
    const uint16_t* idx_key;
    const float* bias_c;
    const float* bias_h;
    uint16_t* entries;
    uint16_t* entry_keys;
    uint16_t* hca_entries;
    const float* norm_c;      // [d] RMS-normalization gain of the CSA entries (nullable)
    const float* norm_h;      // [d] the same for the HCA entries (nullable)
    float eps;
    int* status;
};
// max_span: host bound of each sequence's range length, in the range's own units.
cudaError_t launch_compress_tiles(const TileCompressParams& p, int64_t max_span, cudaStream_t stream);

// Indexer score scan + top-k select.
constexpr int kHistBins = 2048;  // sampled histogram of the prefill select: the top 11 bits of the score key
// histogram of the decode scan and final select: the top kKeyBits bits of the score key (sign,
// exponent and two mantissa bits: bins a quarter of an octave wide).  13 bits were measured slower at
// 1M tokens: the lists get shorter, but the per-bin work of the scan's merge, the threshold search
// and the radix passes grows more than that saves.
constexpr int kKeyBits = 11;
constexpr int kKeyBins = 1 << kKeyBits;
constexpr int kMaxK = 2048;
constexpr int kSegPad = 128;  // keys of slack past each score row in the segment buffer

struct IndexParams {
    const csa_seq* seqs;
    const csa_query* queries;
    int Q, H_I, d_I, m, k;
    const uint16_t* q_idx;    // [Q, H_I, d_I]
    const float* w;           // [Q, H_I]
    const uint16_t* entry_keys;
    const uint8_t* keys_q;      // nullable: 8-bit block-scaled keys [*, d_I] E4M3 (scored instead of entry_keys)
    const uint8_t* key_scales;  // [*, d_I / 32] biased power-of-two exponents of keys_q
    int64_t chunk;            // entries per scan CTA
    int64_t max_entries;      // host bound of floor(L/m) over all queries (grid sizing)
    int64_t e_stride;         // row stride of the score buffer
    int64_t e_seg;            // row stride of the segment buffer (e_stride + 128)
    int max_chunks;           // scan chunks per query the workspace holds (ceil(e_stride / chunk))
    int cand_cap;             // candidate keys a scan chunk may keep
    // workspace
    float* scores;            // [Q, e_stride]
    uint32_t* hist;           // [Q, kKeyBins]; zero before the scan
    uint64_t* seg;            // [Q, e_seg] kept entries (64-bit keys) when they exceed shared memory
    uint32_t* meta;           // [Q, max_chunks] per scan chunk: (threshold bin << 16) | candidate count
    uint32_t* coff;           // [Q, max_chunks + 8] the final select's per-CTA prefixes over chunks (many chunks)
    uint64_t* cand;           // [Q, max_chunks, cand_cap] candidate keys of each chunk, in index order
    // nullable: [Q] words, zero before the scan; the final select sets word q (release) once query
    // q's indices are out, for an attention grid that starts before the select grid ends
    uint32_t* ready;
    int debug_fault;          // 2 (tests of the bounded waits): the select publishes no ready word
    // nullable: [Q, 4] words, zero before the scan.  When set and the scan grid fits the SMs at
    // once (sms: the device's multiprocessor count), the scan grid selects the top-k itself (no
    // final-select launch): its CTAs meet on these per-query counters
    uint32_t* qsync;
    int sms;
    // optional: rows of this cache (row stride prefetch_row_bytes, a multiple of 16) at the selected
    // entries are prefetched into L2 as soon as the selection is known (the attention's gather)
    const unsigned char* prefetch_rows;
    int64_t prefetch_row_bytes;
    // outputs
    int32_t* idx_out;         // [Q, k]
    float* score_out;         // [Q, k] nullable
    int* status;
};
size_t index_ws_bytes(int Q, int64_t e_stride);
size_t index_zero_bytes(int Q);  // leading bytes of the index workspace that must start at zero
// Per-step words of `ws` inside its leading zero bytes, after the histograms: Q ready words (see
// IndexParams::ready), Q item counters (see AttnParams::items_done), then 4 Q scan counters (see
// IndexParams::qsync).
uint32_t* index_ready_words(void* ws, int Q);
// Points the workspace arrays of `p` into `ws` and sets the scan chunking (chunk, max_chunks,
// cand_cap), all derived from (Q, e_stride) exactly as index_ws_bytes sizes them.
void index_ws_carve(IndexParams& p, void* ws, int Q, int64_t e_stride);
// FP4 copies (codes [*, d / 2], scales [*, d / 32]) of the stored bf16 entries [ranges[b][0],
// ranges[b][1]) of the CSA cache (which = 0, ratio m) or the HCA cache (which = 1, ratio m_hca).
cudaError_t launch_quantize_entries(const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries, int which,
                                    int ratio, int d, const uint16_t* entries, uint8_t* entries_q, uint8_t* scales,
                                    int* status, cudaStream_t stream);
// 8-bit block-scaled copies (keys_q [*, d_I] E4M3, scales [*, d_I / 32]) of the stored bf16 indexer
// keys of entries [ranges[b][0], ranges[b][1]) of every sequence.
cudaError_t launch_quantize_keys(const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries, int m,
                                 int d_I, const uint16_t* keys, uint8_t* keys_q, uint8_t* scales, int* status,
                                 cudaStream_t stream);
// Prefill indexer scores as a tensor-core GEMM (d_I = 64, H_I <= 4): chunk rows [0, Qn) are the
// consecutive positions pos0, pos0 + 1, ... of one sequence; row r's causal entries (j < (pos0 + r +
// 1) / m) get scores[r * e_stride + j].
struct PrefillScoreParams {
    const csa_seq* seq;
    const uint16_t* q_idx;   // [Qn, H_I, 64]
    const float* w;          // [Qn, H_I]
    const uint16_t* entry_keys;
    int H_I, m_shift, Qn;     // m = 1 << m_shift
    int64_t pos0;
    int64_t ent_per_cta;     // multiple of 64
    float* scores;
    int64_t e_stride;
    int* status;
};
cudaError_t launch_prefill_scores(const PrefillScoreParams& p, int64_t max_entries, cudaStream_t stream,
                                  bool pdl = false);

// `mid` (nullable): event recorded after the scan kernel (which also selects).
// `sampled`: p.scores already holds the scores (prefill GEMM): no scan, the select kernel takes each
// row's top-k with a sampled threshold; every row must hold at most kSelRowMax entries.
constexpr int64_t kSelRowMax = 32768;
cudaError_t launch_index_topk(IndexParams& p, int64_t max_entries, cudaStream_t stream, bool zero_ws,
                              cudaEvent_t mid = nullptr, bool pdl = false, bool sampled = false);

// Attention over a per-query key list = [selected CSA entries | raw window | HCA entries].
struct AttnParams {
    const csa_seq* seqs;
    const csa_query* queries;
    int Q, H, d;
    const uint16_t* q;          // [Q, H, d]
    const uint16_t* entries;    // CSA entry cache (nullable when k_slots == 0)
    const int32_t* idx;         // [Q, k_slots] (nullable when k_slots == 0)
    int k_slots;
    int m;                      // CSA ratio (bounds check of idx)
    const uint16_t* raw;        // raw latents (window)
    int W;
    const uint16_t* hca;        // HCA cache (nullable when use_hca == 0)
    // FP4 entry caches (E2M1 codes [*, d / 2] and power-of-two block scales [*, d / 32]); when set, the
    // CSA entries / HCA entries are read from these and dequantized into the key tiles
    const uint8_t* entries_q;
    const uint8_t* entries_s;
    const uint8_t* hca_q;
    const uint8_t* hca_s;
    int m_hca;
    int use_hca;
    float scale_log2;           // scale * log2(e)
    const float* sink;          // [H] attention-sink logits (nullable): one more softmax term per head
                                // with a zero value, joined where the query's softmax is complete
    const float* q_norm;        // [d] RMS-normalization gain of every query head (nullable)
    float norm_eps;
    // Items.  n_items == 1: one item covers the whole list (direct output, no merge).  Otherwise
    // items [0, items_front) cut the front part [0, k_slots + W) into chunks of kpi_front keys and
    // items [items_front, n_items) cut the HCA part into chunks of kpi_hca keys; every item writes
    // a partial and combine_kernel merges them.  Chunk sizes are multiples of 64 (one key tile).
    int n_items;
    int items_front;
    int kpi_front;
    int kpi_hca;
    // 1: HCA items do not wait for the preceding launch (griddepcontrol.wait): their inputs (query
    // table, HCA entries) were written two or more launches earlier, which are complete by the time
    // this grid may start.  Only the decode chain sets it.
    int hca_nowait;
    // 1: the query table and the sequence table were written two or more launches back (complete
    // when this grid runs), so they are read before waiting on the previous launch
    int queries_early;
    // 1: one-dimensional grid over all (query, item) pairs with every query's HCA items first, so
    // they take the free SMs before the front items (which wait for the top-k) do.  Launches all
    // items of all queries.
    int hca_first;
    // nullable (multi-item launches): [Q] words the top-k select sets once query q's indices are out;
    // the front items of query q poll theirs instead of waiting for the whole previous grid
    const uint32_t* ready;
    // nullable (multi-item launches): [Q] counters, zero before the launch; every item CTA of query q
    // adds 1 once its partial is stored, and the merge of query q starts when all n_items have
    uint32_t* items_done;
    // > 1: the launch forms thread-block clusters of `cluster` consecutive items of one query (the
    // item counts of both parts are multiples of it); the CTAs of a cluster merge their results
    // through distributed shared memory and store one partial per cluster, so part_o holds
    // n_items / cluster partials per query
    int cluster;
    // 1: full key tiles that are contiguous rows of the HCA cache / of the raw window are loaded by
    // TMA (set by the launcher when the tensor maps could be encoded)
    int tma_hca, tma_x;
    // fault injection for the tests of the bounded waits (csa_debug_inject): 1 = the first loader
    // warp does not arrive on the first key tile's barrier, so the tile never becomes full; wait_ns =
    // the limit of every wait in the kernel
    int debug_fault;
    uint64_t wait_ns;
    // 1: a launch with one item per query (direct outputs) runs one persistent CTA per SM over the
    // queries; q_step is set by the launcher (the grid's CTA count; 0 = one CTA per query)
    int persist;
    int q_step;
    // outputs
    float* out;                 // [Q, H, d]
    float* lse;                 // [Q, H] nullable
    float* part_o;              // [Q, items, 64, d]
    float* part_lse;            // [Q, items, 64]
    int* status;
};
size_t attn_ws_bytes(int Q, int items, int d);
// Point the partial buffers of `p` into `ws` (when n_items > 1).
void attn_ws_carve(AttnParams& p, void* ws);
// Items [item_begin, item_begin + item_count) of every query.
cudaError_t launch_attention_items(const AttnParams& p, int item_begin, int item_count, cudaStream_t stream,
                                   bool pdl = false);
// The log-sum-exp merge of all items' partials (only when n_items > 1).
cudaError_t launch_combine(const AttnParams& p, cudaStream_t stream, bool pdl = false);

// Decode helper: append one token per sequence, compress completed entries, build the query table.
// One thread-block cluster of d/64 CTAs per sequence; CTA s owns channels [64s, 64s + 64).
struct AppendParams {
    csa_seq* seqs;
    int B, append;
    int d, d_I, m, m_hca;
    uint16_t* x;
    uint16_t* logit_c;
    uint16_t* logit_h;
    uint16_t* idx_key;
    const uint16_t* new_rows;  // [B, 3d + d_I] appended token rows to copy into the caches (nullable)
    const float* bias_c;
    const float* bias_h;
    uint16_t* entries;
    uint16_t* entry_keys;
    uint16_t* hca_entries;
    uint8_t* keys_q;         // nullable: 8-bit block-scaled copy of each new indexer key
    uint8_t* key_scales;
    uint8_t* entries_q;      // nullable: FP4 copies of each new CSA / HCA entry (codes, block scales)
    uint8_t* entries_s;
    uint8_t* hca_q;
    uint8_t* hca_s;
    const float* norm_c;     // [d] RMS-normalization gains of new CSA / HCA entries (nullable)
    const float* norm_h;
    float eps;
    csa_query* queries;      // [B] out
    uint32_t* zero_words;    // index workspace words to clear (nullable)
    int64_t n_zero_words;
    int* status;
};
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);

// Prefill helper: query table for positions [p0, p0 + n) of one sequence.
cudaError_t launch_prefill_queries(csa_query* queries, int64_t p0, int64_t n, cudaStream_t stream);

// Address of the device status word on the current device: CSA_OK, or an error code (with the
// message recorded for csa_last_error) when it cannot be looked up.
int device_status(int** out);

// Fault injection state (csa_debug_inject): the fault code and the wait limit in nanoseconds the
// next attention launches use.
void debug_fault_state(int* fault, uint64_t* wait_ns);

// Error reporting shared by entry points defined outside capi.cu.
int validate_dims(const csa_dims* d);             // CSA_OK or the error code (message set)
int set_error(int code, const char* fmt, ...);    // records the message for csa_last_error()

}  // namespace csa

/*
 * csa.h -- C ABI of libcsa: hybrid compressed attention (CSA + HCA) on NVIDIA B200 (sm_100a).
 *
 * The method (sources are web pages, cited by title and section):
 *  - "Frontier Techniques: NTK RoPE, CSA+HCA, QAT, MTP", section 2 "CSA + HCA -- sparse attention
 *    at 1M tokens": CSA compresses every m = 4 tokens into one entry, a Lightning Indexer keeps the
 *    top-1024 entries per query, and attention also covers a 128-token raw sliding window (2.1);
 *    HCA compresses every m' = 128 tokens and attends all of its entries densely (2.2).
 *  - "DeepSeek V4 comprimeix el context: aixi funcionen CSA i HCA": one 512-wide KV latent shared
 *    by all heads (MQA) ("DeepSeek comprimeix la dimensio temporal"); an entry is a softmax-
 *    weighted sum of its tokens with a separate weight per channel (same section); windows
 *    overlap and weights are recomputed per window ("Finestres solapades per evitar fronteres
 *    artificials"); a light indexer scores compressed entries and attention runs over the chosen
 *    ones plus the local window ("CSA: buscar primer i atendre despres"); HCA attends every
 *    128-token summary ("HCA: un resum global 128 vegades mes curt").
 *
 * Readings adopted where the pages are silent (the same readings as the fp64 test oracle):
 *  R1 CSA entry j covers tokens [m*j - m, m*j + m) clipped at 0 (window 2m, overlap m); HCA entry j
 *     covers [m'*j, m'*j + m').  Entry j exists once m*(j+1) <= L.
 *  R2 z_t[c] = logit_t[c] + bias[t - start_j][c], start_j the unclipped window start; weights are a
 *     softmax over the window per channel; entry = sum_t w_t * x_t; indexer key (channels
 *     c < d_I) = sum_t w_t * idx_key_t[c] with the same weights.
 *  R3 indexer score s_j = sum_h w_h * relu(q^I_h . K^I_j) (no scale); top-k by score descending,
 *     ties to the lower entry index; fewer than k causal entries selects all and pads with -1.
 *  R4 a query at visible length L sees raw tokens [0, L): CSA entries j < floor(L/m), HCA entries
 *     j < floor(L/m'), and the raw window [max(0, L-W), L).
 *  R5 K = V = the stored bf16 vector; logits scaled by `scale` (1/sqrt(d)); the CSA partial
 *     (selected entries + window) and the HCA partial are merged by log-sum-exp; the window is
 *     counted once (in the CSA partial).
 *
 * Conventions shared by every call:
 *  - bf16 data is passed as csa_bf16 (the raw 16-bit pattern); all tensors are dense row-major.
 *  - Every pointer argument is DEVICE memory owned by the caller, except `dims` and `args`
 *    structs, which are read on the host during the call.  The library never allocates device
 *    memory: scratch space is the caller's `ws` buffer of at least csa_workspace_size() bytes
 *    (256-byte aligned).  The workspace holds no state between calls.
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream) and never synchronize
 *    the host.  They may be captured in CUDA graphs.
 *  - Return codes: CSA_OK, or a negative CSA_ERR_* when host-side validation or the launch fails
 *    (then nothing, or only part of the work, was enqueued; csa_last_error() has the reason).
 *    Data-dependent errors found on the device (an out-of-range entry index, a wait that timed
 *    out) set a device status word instead, which csa_sync_status() returns; the affected
 *    element is skipped, never read out of bounds.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t csa_bf16;
typedef struct CUstream_st* csa_stream_t;

#define CSA_OK 0
#define CSA_ERR_ARG (-1)         /* invalid argument (null pointer, bad size, misalignment) */
#define CSA_ERR_UNSUPPORTED (-2) /* a size outside what the kernels implement */
#define CSA_ERR_CUDA (-3)        /* a CUDA launch or runtime call failed */
#define CSA_ERR_TIMEOUT (-4)     /* device: a bounded wait inside a kernel ran out */
#define CSA_ERR_INDEX (-5)       /* device: an entry index or length was out of range */

/* Widths of one hybrid attention layer.  Supported: d in {128, 512}; 1 <= H <= 64;
 * d_I in {32, 64}; 1 <= H_I <= 8; m in {1, 2, 4, 8}; m_hca in {1..1024}; 1 <= k <= 2048;
 * 0 <= W <= 4096. */
typedef struct csa_dims {
    int32_t d;     /* KV latent width (keys = values = latent) */
    int32_t H;     /* query heads sharing the latent (MQA) */
    int32_t d_I;   /* indexer key width */
    int32_t H_I;   /* indexer heads */
    int32_t m;     /* CSA compression ratio (window 2m, overlapping) */
    int32_t m_hca; /* HCA compression ratio (window m', non-overlapping) */
    int32_t k;     /* CSA entries selected per query */
    int32_t W;     /* raw sliding window, in tokens */
} csa_dims;

/* Where one sequence lives inside the (ragged, packed) caches.  Device memory. */
typedef struct csa_seq {
    int64_t tok_off; /* row of token 0 in the raw arrays x, logit_c, logit_h ([*, d]), idx_key ([*, d_I]) */
    int64_t csa_off; /* row of CSA entry 0 in entries ([*, d]) and entry_keys ([*, d_I]) */
    int64_t hca_off; /* row of HCA entry 0 in hca_entries ([*, d]) */
    int64_t len;     /* raw tokens currently held, L */
} csa_seq;

/* One query: its sequence and its visible length L (the query sees raw tokens [0, L)).
 * Device memory.  Precondition: seq indexes an entry of the csa_seq table passed with it.  The
 * calls are not given the table's length, so they cannot check the upper bound; a negative seq or a
 * non-zero `reserved` is reported as CSA_ERR_INDEX and the query is skipped. */
typedef struct csa_query {
    int32_t seq;      /* index into the csa_seq table, 0 <= seq < number of sequences */
    int32_t reserved; /* must be 0 */
    int64_t len;      /* visible length L, 1 <= L <= seqs[seq].len */
} csa_query;

/* f3 -- optional normalization and sink parameters of a layer ("DeepSeek V4 comprimeix el context",
 * "CSA: buscar primer i atendre despres", last paragraph: queries and compressed entries are
 * normalized to stabilize the logits, and learned attention-sink logits absorb excess attention).
 * Read on the host during a call; every pointer is device memory (fp32, 16-byte aligned) or NULL,
 * which turns that part off.
 *  q_norm:       [d] gain of the RMS normalization of each query head, q / sqrt(mean q^2 + eps) *
 *                gain, applied before the logits (the normalized query is rounded to bf16).
 *  entry_norm_c: [d] gain of the same normalization of every CSA entry as it is compressed (the
 *                stored entry, key and value of the attention, is the normalized one); the raw
 *                window and the indexer keys are not normalized.  Needs m = 4.
 *  entry_norm_h: [d] the same for the HCA entries.  Needs m_hca a power of two from 4 to 128.
 *  sink:         [H] the sink logit z_h of each head: one more term of the head's (merged) softmax
 *                with a zero value, lse' = log(e^lse + e^z), out' = out * e^(lse - lse').
 *  eps:          the normalization's epsilon. */
typedef struct csa_norms {
    const float* q_norm;
    const float* entry_norm_c;
    const float* entry_norm_h;
    const float* sink;
    float eps;
    int32_t reserved; /* must be 0 */
} csa_norms;

/* a1/a2 -- token-axis compressor ("DeepSeek V4 comprimeix el context", sections "DeepSeek
 * comprimeix la dimensio temporal" and "Finestres solapades per evitar fronteres artificials";
 * "Frontier Techniques", 2.1 and 2.2).
 *  which = 0: CSA (ratio dims->m, window 2m, rows at seqs[b].csa_off, also writes entry_keys if
 *             non-NULL from idx_key); which = 1: HCA (ratio dims->m_hca, window m', rows at
 *             seqs[b].hca_off; idx_key/entry_keys must be NULL).
 *  ranges: device int64 [B][2]; sequence b recomputes entries [ranges[b][0], ranges[b][1]).
 *          Entries must be complete: m*ranges[b][1] <= seqs[b].len (else CSA_ERR_INDEX on device).
 *  max_entries: host-side upper bound of ranges[b][1] - ranges[b][0] (sizes the grid).
 *  x, logit: [*, d] bf16 rows addressed by seqs[b].tok_off; bias: fp32 [win, d].
 *  Outputs entries/entry_keys are bf16 (round-to-nearest-even of fp32 accumulations). */
int csa_compress(const csa_dims* dims, int which, const csa_seq* seqs, const int64_t* ranges, int B,
                 int64_t max_entries, const csa_bf16* x, const csa_bf16* logit, const float* bias,
                 const csa_bf16* idx_key, csa_bf16* entries, csa_bf16* entry_keys, csa_stream_t stream);

/* a1 + a2 in one pass -- both caches for token ranges ("DeepSeek V4 comprimeix el context", sections
 * "DeepSeek comprimeix la dimensio temporal" and "Finestres solapades per evitar fronteres
 * artificials"; "HCA: un resum global 128 vegades mes curt"; "Frontier Techniques", 2.1 and 2.2).
 * For sequence b with tok_ranges[b] = [t0, t1) (device int64 [B][2], t1 <= seqs[b].len): every CSA
 * entry j in [t0/m, t1/m) with its indexer key, and every HCA entry in [t0/m_hca, t1/m_hca), i.e. the
 * entries whose last token lies in [t0, t1).  With m = 4 and m_hca a power of two from 4 to 128 each
 * raw row (x, both logit arrays, idx_key) is read once for both caches; other ratios run the two
 * caches one after the other.  max_tokens: host bound of t1 - t0 over the sequences (sizes the
 * grid).  Entries equal those of csa_compress and of the decode append bit for bit.  norms (host
 * struct, nullable): only entry_norm_c / entry_norm_h / eps are used (normalized entries; csa_compress
 * has no normalization).  A range outside [0, seqs[b].len] is reported as CSA_ERR_INDEX on the device. */
int csa_compress_all(const csa_dims* dims, const csa_seq* seqs, const int64_t* tok_ranges, int B, int64_t max_tokens,
                     const csa_bf16* x, const csa_bf16* logit_c, const csa_bf16* logit_h, const float* bias_c,
                     const float* bias_h, const csa_bf16* idx_key, csa_bf16* entries, csa_bf16* entry_keys,
                     csa_bf16* hca_entries, const csa_norms* norms, csa_stream_t stream);

/* a3/a4 -- Lightning-Indexer scores and top-k ("Frontier Techniques", 2.1; "DeepSeek V4
 * comprimeix el context", "CSA: buscar primer i atendre despres").  For query i at length L:
 * s_j = sum_h w[i][h] * relu(q_idx[i][h] . entry_keys[csa_off + j]) over j < floor(L/m); the k
 * best by (score desc, index asc) are written to idx_out[i][0..k) in ascending index order, -1 past
 * the end.  score_out (nullable): the fp32 score of each written index (NaN past the end).
 *  q_idx: bf16 [Q, H_I, d_I]; w: fp32 [Q, H_I]; max_len: host bound of every query's L. */
int csa_index_topk(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                   const csa_bf16* q_idx, const float* w, const csa_bf16* entry_keys, int32_t* idx_out,
                   float* score_out, void* ws, size_t ws_bytes, csa_stream_t stream);

/* f1 -- 8-bit block-scaled indexer keys ("Frontier Techniques", section 3: the indexer's QK path is
 * quantized to a block-scaled format; "Compressed attention", sections 3-4: block scales carry
 * bytes).  Each 32-channel block of a key shares one power-of-two scale 2^e, stored as the byte
 * e + 127, where 2^e is the smallest power of two with amax <= 448 * 2^e (a zero block: e = -127);
 * the block's elements are FP8 E4M3 bytes of x / 2^e rounded to nearest even.  Rows follow the
 * CSA entry rows (keys_q row csa_off + j holds entry j's d_I bytes, key_scales row csa_off + j its
 * d_I / 32 scale bytes).  Per entry 64 + 2 bytes instead of 128 at d_I = 64.
 *
 * csa_quantize_keys: the 8-bit copies of the stored bf16 keys of entries [ranges[b][0],
 * ranges[b][1]) of every sequence (ranges and max_entries as csa_compress; the entries must
 * exist: m * ranges[b][1] <= seqs[b].len, else CSA_ERR_INDEX on the device).
 * csa_index_topk_mx8: csa_index_topk scoring the dequantized 8-bit keys (queries stay bf16):
 * s_j = sum_h w_h relu(q_idx_h . K_j), K_j[c] = 2^e * E4M3 value; same outputs, same workspace
 * size (CSA_OP_INDEX_TOPK). */
int csa_quantize_keys(const csa_dims* dims, const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries,
                      const csa_bf16* entry_keys, uint8_t* keys_q, uint8_t* key_scales, csa_stream_t stream);
int csa_index_topk_mx8(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                       const csa_bf16* q_idx, const float* w, const uint8_t* keys_q, const uint8_t* key_scales,
                       int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes, csa_stream_t stream);

/* a5 -- sparse MQA attention over the selected CSA entries plus the raw window ("DeepSeek V4
 * comprimeix el context", "CSA: buscar primer i atendre despres"; "Frontier Techniques", 2.1).
 * Keys (= values): entries[csa_off + idx[i][s]] for every s with idx[i][s] >= 0, then
 * x[tok_off + t] for t in [max(0, L-W), L).  For every head h:
 *   out[i][h] = softmax_keys(scale * q[i][h] . key) @ keys,  lse[i][h] = logsumexp(scale * q . key).
 * An index >= floor(L/m) is skipped and reported as CSA_ERR_INDEX.
 *  q: bf16 [Q, H, d]; idx: int32 [Q, k]; out: fp32 [Q, H, d]; lse: fp32 [Q, H] (nullable). */
int csa_sparse_attn(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, const csa_bf16* q,
                    const csa_bf16* entries, const int32_t* idx, const csa_bf16* x, float scale, float* out,
                    float* lse, void* ws, size_t ws_bytes, csa_stream_t stream);

/* f4 -- FP4 compressed entries with block scales ("Compressed attention · CSA / HCA", section 3: the
 * FP4 KV cache of V4.1 carries block scales and a packing overhead).  Each 32-channel block of an
 * entry row shares one power-of-two scale 2^e, stored as the byte e + 127, where 2^e is the smallest
 * power of two with amax <= 6 * 2^e (a zero block: e = -127); the elements are E2M1 codes (sign, two
 * exponent bits with bias 1, one mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) of x / 2^e
 * rounded to nearest even, two per byte, the even channel in the low nibble.  Row r of an FP4 cache
 * mirrors row r of its bf16 cache (CSA: csa_off + j, HCA: hca_off + j): d / 2 code bytes
 * (entries_q, 16-byte aligned) and d / 32 scale bytes (entry_scales).  Per 512-wide entry 256 + 16
 * bytes instead of 1,024.  The attention uses the dequantized entries (code * 2^e, every one a bf16
 * value) as keys and values; the raw window stays bf16.
 *
 * csa_quantize_entries: the FP4 copies of the stored bf16 entries [ranges[b][0], ranges[b][1]) of
 * every sequence's CSA cache (which = 0) or HCA cache (which = 1); ranges and max_entries as in
 * csa_compress (the entries must exist, else CSA_ERR_INDEX on the device).
 * csa_sparse_attn_fp4 / hca_dense_attn_fp4: csa_sparse_attn / hca_dense_attn reading the entries
 * from the FP4 caches; same outputs and workspace sizes. */
int csa_quantize_entries(const csa_dims* dims, const csa_seq* seqs, const int64_t* ranges, int B, int64_t max_entries,
                         int which, const csa_bf16* entries, uint8_t* entries_q, uint8_t* entry_scales,
                         csa_stream_t stream);
int csa_sparse_attn_fp4(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, const csa_bf16* q,
                        const uint8_t* entries_q, const uint8_t* entry_scales, const int32_t* idx, const csa_bf16* x,
                        float scale, float* out, float* lse, void* ws, size_t ws_bytes, csa_stream_t stream);
int hca_dense_attn_fp4(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                       const csa_bf16* q, const uint8_t* hca_q, const uint8_t* hca_scales, const csa_bf16* x, int W,
                       float scale, float* out, float* lse, void* ws, size_t ws_bytes, csa_stream_t stream);

/* a6 -- dense MQA attention over every visible HCA entry ("Frontier Techniques", 2.2; "DeepSeek V4
 * comprimeix el context", "HCA: un resum global 128 vegades mes curt").  Keys: hca_entries[hca_off
 * + j] for j < floor(L/m_hca), then (when W > 0) the raw window [max(0, L-W), L).  An empty key set
 * gives lse = -inf and out = 0.  max_len: host bound of every query's L. */
int hca_dense_attn(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q, int64_t max_len,
                   const csa_bf16* q, const csa_bf16* hca_entries, const csa_bf16* x, int W, float scale,
                   float* out, float* lse, void* ws, size_t ws_bytes, csa_stream_t stream);


/* Arguments of one decode step of B sequences (all pointers device memory). */
typedef struct csa_decode_args {
    csa_dims dims;
    int32_t B;
    int32_t append;      /* 1: every sequence first takes one new token; len += 1 and the entries
                            that this token completes are compressed.  The token's rows at
                            tok_off + len are either already written in x/logit_c/logit_h/idx_key by
                            the caller (new_rows = NULL) or copied there from new_rows */
    int64_t max_len;     /* host bound of every sequence's len after the append (sizes grids) */
    float scale;         /* logit scale, normally 1/sqrt(d) */
    csa_seq* seqs;       /* [B]; len is updated in place when append = 1 */
    csa_bf16* x;             /* raw latents [*, d] (written only when new_rows is given) */
    csa_bf16* logit_c;       /* CSA compressor logits [*, d] (idem) */
    csa_bf16* logit_h;       /* HCA compressor logits [*, d] (idem) */
    csa_bf16* idx_key;       /* raw indexer keys [*, d_I] (idem) */
    const float* bias_c;     /* [2m, d] */
    const float* bias_h;     /* [m_hca, d] */
    csa_bf16* entries;       /* CSA entry cache [*, d] */
    csa_bf16* entry_keys;    /* CSA indexer-key cache [*, d_I] */
    csa_bf16* hca_entries;   /* HCA entry cache [*, d] */
    const csa_bf16* q;       /* [B, H, d] */
    const csa_bf16* q_idx;   /* [B, H_I, d_I] */
    const float* w;          /* [B, H_I] */
    float* out;              /* [B, H, d] merged output */
    float* lse;              /* [B, H] merged log-sum-exp (nullable) */
    int32_t* idx_out;        /* [B, k] selected entries (nullable) */
    const csa_bf16* new_rows; /* [B, 3d + d_I]: x | logit_c | logit_h | idx_key of each sequence's
                                 appended token, copied into the caches by the call (append = 1;
                                 16-byte aligned rows), or NULL */
    uint8_t* keys_q;          /* optional 8-bit block-scaled indexer keys [*, d_I] (see
                                 csa_quantize_keys; 16-byte aligned), or NULL.  When given, the
                                 indexer scores these instead of entry_keys, and the append also
                                 writes the 8-bit copy of every key it completes */
    uint8_t* key_scales;      /* their block scales [*, d_I / 32] (2-byte aligned), with keys_q */
    const int32_t* idx_in;    /* optional [B, k]: a selection reused from another layer of the same
                                 sequences (cross-layer index reuse, "Compressed attention", sections
                                 1 and 5: consecutive layers may share the selected-position table,
                                 and the reusing layer must read the source layer's selection).
                                 When given, this call runs no indexer (q_idx and w may be NULL,
                                 idx_out must be NULL) and attends these entries of its own CSA
                                 cache; entries are named by their position j, which is the same in
                                 every layer of a sequence */
    const csa_norms* norms;   /* optional (host struct, see csa_norms): query / entry normalization
                                 and sink logits; NULL: none */
    uint8_t* entries_q;       /* optional FP4 copy of the CSA entry cache [*, d / 2] (see
                                 csa_quantize_entries; 16-byte aligned), with entry_scales [*, d / 32],
                                 hca_q and hca_scales (all four or none; m = 4 and m_hca a power of two
                                 from 4 to 128).  When given, the attention reads the FP4 caches and
                                 the append also writes the FP4 copy of every entry it completes */
    uint8_t* entry_scales;
    uint8_t* hca_q;           /* optional FP4 copy of the HCA entry cache [*, d / 2] (16-byte aligned) */
    uint8_t* hca_scales;      /* [*, d / 32] */
} csa_decode_args;

/* a8 + a3..a7 -- one decode step: optional append (and the compressor updates it triggers), then
 * for every sequence one query at L = len: indexer top-k, sparse CSA attention with the window,
 * dense HCA attention (window excluded), merged by log-sum-exp. */
int hybrid_attn_decode(const csa_decode_args* args, void* ws, size_t ws_bytes, csa_stream_t stream);

/* Arguments of a causal prefill of one sequence (all pointers device memory). */
typedef struct csa_prefill_args {
    csa_dims dims;
    int32_t compress;        /* 1: first compress every CSA and HCA entry complete in [0, q_end) */
    int32_t reserved;
    int64_t len;             /* host copy of seq->len (>= q_end) */
    int64_t q_begin, q_end;  /* query positions to compute; position p sees L = p + 1 tokens */
    float scale;
    const csa_seq* seq;      /* [1] */
    const csa_bf16* x;
    const csa_bf16* logit_c;
    const csa_bf16* logit_h;
    const csa_bf16* idx_key;
    const float* bias_c;
    const float* bias_h;
    csa_bf16* entries;
    csa_bf16* entry_keys;
    csa_bf16* hca_entries;
    const csa_bf16* q;       /* [q_end - q_begin, H, d] */
    const csa_bf16* q_idx;   /* [q_end - q_begin, H_I, d_I] */
    const float* w;          /* [q_end - q_begin, H_I] */
    float* out;              /* [q_end - q_begin, H, d] */
    float* lse;              /* [q_end - q_begin, H] (nullable) */
    int32_t* idx_out;        /* [q_end - q_begin, k] (nullable) */
    const int32_t* idx_in;   /* optional [q_end - q_begin, k]: a selection reused from another layer
                                (as in csa_decode_args): no indexer runs; q_idx / w may be NULL and
                                idx_out must be NULL */
    const csa_norms* norms;  /* optional (host struct): as in csa_decode_args; the entry
                                normalization applies to the compress step (compress = 1) */
} csa_prefill_args;

/* a1, a2 full pass + a3..a7 for every query position in [q_begin, q_end) of one sequence.
 * The positions run in chunks of 64 queries per multiprocessor of the current device (environment
 * CSA_PREFILL_CHUNK overrides it); the workspace holds one chunk's score rows, about
 * 4 B x chunk x floor(q_end / m), so query its size (CSA_OP_PREFILL) on the device that runs the call:
 * a workspace smaller than the call's plan is rejected with CSA_ERR_ARG. */
int hybrid_attn_prefill(const csa_prefill_args* args, void* ws, size_t ws_bytes, csa_stream_t stream);

/* Workspace sizes.  `op` selects the call and `args` points to the arguments it describes:
 *   CSA_OP_INDEX_TOPK:  csa_ws_query {dims, Q, max_len}
 *   CSA_OP_SPARSE_ATTN: csa_ws_query {dims, Q, max_len}
 *   CSA_OP_HCA_ATTN:    csa_ws_query {dims, Q, max_len}
 *   CSA_OP_DECODE:      csa_decode_args
 *   CSA_OP_PREFILL:     csa_prefill_args
 * Returns 0 for an unknown op or invalid arguments. */
#define CSA_OP_INDEX_TOPK 1
#define CSA_OP_SPARSE_ATTN 2
#define CSA_OP_HCA_ATTN 3
#define CSA_OP_DECODE 4
#define CSA_OP_PREFILL 5

typedef struct csa_ws_query {
    csa_dims dims;
    int32_t Q;
    int32_t reserved;
    int64_t max_len;
} csa_ws_query;

size_t csa_workspace_size(int op, const void* args);

/* Message of the last error returned on the calling host thread ("" if none). */
const char* csa_last_error(void);

/* Synchronizes `stream`, then returns and clears the device status word of the current device
 * (CSA_OK, CSA_ERR_INDEX or CSA_ERR_TIMEOUT), or CSA_ERR_CUDA if synchronization failed. */
int csa_sync_status(csa_stream_t stream);

/* Per-stage timing of hybrid_attn_decode (a profiling aid; off by default).  With a non-NULL
 * array of `count` cudaEvent_t handles (created by the caller, owned by the caller), every later
 * hybrid_attn_decode call on this host thread records CSA_DECODE_MARKS consecutive events of the
 * array, cyclically from index 0, on its stream: before the append kernel, after it, after the
 * indexer (the score scan, whose last CTA per query also selects the top-k), again at the same point
 * (the select has no kernel of its own), after attention (and its merge).  Inside a stream
 * capture the records become graph nodes.  NULL / 0 turns it off.  Returns CSA_OK or CSA_ERR_ARG
 * (count not a positive multiple of CSA_DECODE_MARKS). */
#define CSA_DECODE_MARKS 5
int csa_set_stage_events(void* const* events, int count);

/* csa_index_topk without a workspace argument (no counterpart in the pages: it only changes where
 * the scratch lives).  For callers that cannot provide device memory at call time -- code under a
 * framework whose allocator owns all device buffers, loops that must not allocate once running, or
 * bindings that only see input and output pointers.  The scratch is a fixed array inside the
 * library, about 14.2 MiB on every device that loads it, held until the process exits.
 * Limits: Q <= 16 and Q * ceil4(floor(max_len / m)) <= 1,048,576; larger calls return
 * CSA_ERR_UNSUPPORTED with a message and enqueue nothing.  It never allocates or frees memory.
 * The first call on a device looks up the array's device address (once per device, with that
 * device current); make that first call before any stream capture.  All calls on a device share
 * the one array, so calls whose kernels overlap on the GPU (different streams, or concurrent
 * graph replays) race: serialize them.  Each call clears the parts that must start at zero.
 * Arguments, results and device-side errors are those of csa_index_topk. */
int csa_index_topk_noalloc(const csa_dims* dims, const csa_seq* seqs, const csa_query* queries, int Q,
                           int64_t max_len, const csa_bf16* q_idx, const float* w, const csa_bf16* entry_keys,
                           int32_t* idx_out, float* score_out, csa_stream_t stream);

/* Fault injection for testing the bounded waits (a test aid; off by default; no counterpart in the
 * pages).  Every wait inside a kernel gives up after a time limit, records CSA_ERR_TIMEOUT in the
 * device status word and lets the kernel wind down (the CTA waits for its own copies in flight,
 * frees its tensor memory and exits), so a fault never hangs the device.  fault = 1 makes the
 * attention kernel's first loader warp skip its arrival on the first key tile of every CTA, so that
 * tile never becomes full and the waits on it run out; fault = 2 makes the top-k select of
 * hybrid_attn_decode publish no per-query ready word, so the front attention items' waits on those
 * words run out; fault = 0 turns injection off.
 * wait_limit_ns > 0 sets the limit of the attention kernel's waits (0 restores the default of 2 s).
 * Process-wide; applies to launches issued after the call.  Returns CSA_OK or
 * CSA_ERR_ARG. */
int csa_debug_inject(int fault, int64_t wait_limit_ns);

/* Library version, major * 10000 + minor * 100 + patch. */
int csa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H */

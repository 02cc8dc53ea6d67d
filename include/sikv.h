/*
 * sikv.h -- C ABI of libsikv, the Self-Indexing KVCache decode hot path on
 * NVIDIA B200 (sm_100a).
 *
 * Method: "Self-Indexing KVCache: Predicting Sparse Attention from Compressed
 * Keys" (summary page at gist.science, paper 2603.14224), technical summary,
 * cited below as [SIKV 2.1.n] for item n of its section 2.1 (core components):
 *   2.1.1  sign-based 1-bit vector quantization of the keys: channel-mean
 *          ("entropy-aware") normalization, 4-dim sub-vectors whose sign
 *          pattern picks one of 16 clusters, a codebook built in one pass;
 *          the code both reconstructs the key and indexes it for retrieval;
 *   2.1.2  compressed-domain top-k retrieval by LUT-GEMV: the query is split
 *          like the key, each sub-query is dotted with the 16 centroids of its
 *          subspace, and a token's score sums the table entries its codes pick;
 *   2.1.3  token-wise code layout (random access per token) and 64
 *          full-precision sink tokens kept from prefill;
 *   2.1.4  dequantization fused with the sparse attention pass.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates device memory.  Its only global state is (a) per-device
 *    launch facts computed on the first call on each device (a kernel's
 *    shared-memory limit, its occupancy and cluster occupancy, each written
 *    once with the same value by any thread) and (b) the fixed scratch array
 *    of sikv_sparse_attn_static with its per-device address cache.  Every
 *    call only enqueues kernels on `stream` and returns without synchronizing.
 *  - Scratch memory comes from the caller's `workspace` (device, 256-byte
 *    aligned, at least sikv_*_workspace_size() bytes).  Zero the whole
 *    workspace once before first use (sikv_workspace_init): its first 256
 *    bytes hold a sticky device status word (read and cleared with
 *    sikv_check_device_status), and sikv_decode keeps per-segment counters
 *    there that every call leaves at zero again.
 *  - Layouts (row-major, contiguous), with B = batch, Hq / Hkv = query / KV
 *    heads, G = Hq / Hkv (query heads per KV head; query head h*G+g belongs to
 *    KV head h), D = head_dim = 128, P = D/4 = 32 subspaces, Nmax =
 *    max_seq_len, S = num_sinks, kmax = max_topk:
 *      K, V       [B][Hkv][Nmax][D]      dtype (fp32 or bf16)
 *      q, out     [B][Hq][D]             dtype
 *      mu         [B][Hkv][D]            fp32   channel means
 *      codes      [B][Hkv][Nmax][D/8]    uint8  16 bytes per token
 *      codebook   [B][Hkv][P][16][4]     fp32   centroids of k - mu
 *      counts     [B][Hkv][P][16]        int32  cluster sizes
 *      scores     [B][Hkv][Nmax]         fp32
 *      idx        [B][Hkv][kmax]         int32  selected token positions
 *      seq_lens   [B]                    int32  N_b, 0 <= N_b <= Nmax (device)
 *      k_per_seq  [B]                    int32  k_b, 0 <= k_b <= min(kmax, max(N_b - S, 0)) (device)
 *    Rows past N_b are neither read nor written.
 *  - Sinks are tokens [0, min(S, N_b)).  Tokens [S, N_b) are the scored,
 *    "compressed" tokens; n_b = max(N_b - S, 0) of them.
 *  - Code byte m of a token holds the code of subspace 2m in its low nibble
 *    and of subspace 2m+1 in its high nibble; bit i of a code is
 *    [k[4s+i] >= mu[4s+i]] (a tie gives 1).
 *  - Host-side argument errors return a status and launch nothing.  Errors
 *    that only the device can see (a seq_len, k or index out of range) set a
 *    bit of the device status word (SIKV_DEVERR_*), and the offending unit of
 *    work is skipped; kernels never trap.
 */
#ifndef SIKV_H
#define SIKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SIKV_API __attribute__((visibility("default")))
#else
#define SIKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *sikv_stream_t;

typedef enum sikv_status {
    SIKV_OK = 0,
    SIKV_ERR_INVALID_ARG = 1,   /* null pointer, bad shape or size */
    SIKV_ERR_UNSUPPORTED = 2,   /* head_dim != 128, group > 8, unknown dtype, misalignment */
    SIKV_ERR_WORKSPACE = 3,     /* workspace null, misaligned or too small */
    SIKV_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    SIKV_ERR_DEVICE = 5         /* the device status word holds an error */
} sikv_status;

typedef enum sikv_dtype {
    SIKV_DTYPE_F32 = 0,
    SIKV_DTYPE_BF16 = 1
} sikv_dtype;

/* Bits of the device status word. */
#define SIKV_DEVERR_SEQ_LEN 0x1   /* seq_lens[b] < 0 or > max_seq_len */
#define SIKV_DEVERR_TOPK 0x2      /* k_per_seq[b] < 0, > max_topk or > max(N_b - S, 0) */
#define SIKV_DEVERR_INDEX 0x4     /* a selected index outside [S, N_b) */
#define SIKV_DEVERR_TIMEOUT 0x8   /* a bounded wait between the CTAs of a segment ran out */
#define SIKV_DEVERR_APPEND 0x10   /* append rows [start_b, start_b + count_b) outside [0, max_seq_len) */

typedef struct sikv_params {
    int32_t dtype;          /* sikv_dtype of K, V, q and out */
    int32_t batch;          /* B >= 1 */
    int32_t num_q_heads;    /* Hq, a multiple of num_kv_heads */
    int32_t num_kv_heads;   /* Hkv >= 1; G = Hq / Hkv must be <= 8 */
    int32_t head_dim;       /* D; only 128 is supported */
    int32_t max_seq_len;    /* Nmax >= 1: row capacity of K, V, codes, scores */
    int32_t num_sinks;      /* S >= 0 (the pages keep 64) */
    int32_t max_topk;       /* kmax >= 0: row capacity of idx */
    float softmax_scale;    /* <= 0 selects 1/sqrt(D) */
    int32_t decode_path;    /* sikv_decode_path: which kernels sikv_decode runs (0: automatic) */
    int32_t reserved[2];    /* must be 0 */
} sikv_params;

/*
 * Kernels of one sikv_decode / sikv_decode_qv / sikv_decode_host step.  Every
 * path computes the same result (identical scores, identical selection; the
 * attention differs only by fp32 summation order).  AUTO picks the first that
 * applies to the shape, in this order; a forced path that does not apply
 * returns SIKV_ERR_UNSUPPORTED.
 *  - CLUSTER: one launch; the CTAs of each (sequence, KV head) segment form a
 *    thread-block cluster (at most 16 CTAs of 16384 tokens: Nmax <= 262144)
 *    and agree through distributed shared memory.  Any batch size: clusters
 *    that do not fit at once run in later waves.
 *  - COOPERATIVE: one cooperative launch per group of sequences whose CTAs all
 *    fit on the device at once; the CTAs of a segment agree through counters
 *    in the workspace.  Any Nmax.
 *  - COMPOSED: sikv_score, sikv_topk and sikv_sparse_attn's kernels.
 */
typedef enum sikv_decode_path {
    SIKV_DECODE_AUTO = 0,
    SIKV_DECODE_CLUSTER = 1,
    SIKV_DECODE_COOPERATIVE = 2,
    SIKV_DECODE_COMPOSED = 3
} sikv_decode_path;

/* Library version as 10000*major + 100*minor + patch. */
SIKV_API int32_t sikv_version(void);

/* Human-readable name of a status code (static storage). */
SIKV_API const char *sikv_status_string(sikv_status status);

/* Zero the whole workspace; enqueued on `stream`.  Call once per workspace. */
SIKV_API sikv_status sikv_workspace_init(void *workspace, size_t workspace_bytes, sikv_stream_t stream);

/* Synchronize `stream`, copy the device status word to *device_flags (may be
 * NULL) and clear it.  Returns SIKV_ERR_DEVICE if any flag was set. */
SIKV_API sikv_status sikv_check_device_status(void *workspace, size_t workspace_bytes,
                                     sikv_stream_t stream, int32_t *device_flags);

/* Workspace bytes each entry point needs for these parameters (0 on bad params). */
SIKV_API size_t sikv_encode_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_score_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_topk_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_sparse_attn_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_decode_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_decode_host_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_append_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_dense_attn_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_kmeans_workspace_size(const sikv_params *p);
SIKV_API size_t sikv_quantize_values_workspace_size(const sikv_params *p);

/* Number of kernels one sikv_decode call enqueues for these parameters
 * (0 on bad params, or when the forced decode_path does not apply). */
SIKV_API int32_t sikv_decode_launches(const sikv_params *p);

/* The sikv_decode_path (CLUSTER, COOPERATIVE or COMPOSED) that one
 * sikv_decode call with these parameters runs on the current device: the
 * automatic choice resolved, or the forced path; 0 on bad params or when a
 * forced path does not apply.  Queries occupancy once per device. */
SIKV_API int32_t sikv_decode_resolved_path(const sikv_params *p);

/*
 * sikv_encode_keys -- prefill encoder [SIKV 2.1.1, 2.1.3].
 *
 * For every (b, h):
 *   mu[c]       = mean of K[t][c] over t in [S, N_b), computed exactly and
 *                 rounded once to fp32 (0 when N_b <= S);
 *   codes[t]    = packed sign-pattern codes of every token t in [0, N_b)
 *                 (sink rows are written too and never used);
 *   codebook    = c[s][j] = mean over t in [S, N_b) with code_s(t) == j of
 *                 K[t][4s:4s+4] - mu[4s:4s+4]; 0 for an empty cluster;
 *   counts      = cluster sizes (optional output, may be NULL).
 * Inputs: K (dtype), seq_lens.  Outputs: mu, codes, codebook, counts.
 * The workspace holds per-chunk partial sums.  Its size depends on the
 * current device: the chunk length is chosen so that the chunk CTAs fill
 * whole waves of its SMs, so query the size on the device that runs the call.
 */
SIKV_API sikv_status sikv_encode_keys(const sikv_params *p, const void *K, const int32_t *seq_lens,
                             float *mu, uint8_t *codes, float *codebook, int32_t *counts,
                             void *workspace, size_t workspace_bytes, sikv_stream_t stream);

/*
 * sikv_score -- compressed-domain LUT-GEMV scoring [SIKV 2.1.2].
 *
 * For every (b, h): q_bar = sum of the G query rows of the group;
 * LUT[s][j] = q_bar[4s:4s+4] . c[s][j]; scores[t] = sum_s LUT[s][code_s(t)]
 * + q_bar . mu for t in [S, N_b), and -inf for t in [0, min(S, N_b)).
 * Computed in fp32.  Inputs: q, codes, codebook, mu, seq_lens.
 */
SIKV_API sikv_status sikv_score(const sikv_params *p, const void *q, const uint8_t *codes,
                       const float *codebook, const float *mu, const int32_t *seq_lens,
                       float *scores, void *workspace, size_t workspace_bytes,
                       sikv_stream_t stream);

/*
 * sikv_topk -- exact top-k of the compressed-domain scores [SIKV 2.1.2].
 *
 * For every (b, h): the k_b tokens t in [S, N_b) that come first in the
 * order (score descending, t ascending); -0.0 equals +0.0.  idx[b][h][0..k_b)
 * receives them in ascending token order and idx[b][h][k_b..kmax) is set to
 * -1.  Scores must not be NaN.  Inputs: scores, seq_lens, k_per_seq.
 */
SIKV_API sikv_status sikv_topk(const sikv_params *p, const float *scores, const int32_t *seq_lens,
                      const int32_t *k_per_seq, int32_t *idx, void *workspace,
                      size_t workspace_bytes, sikv_stream_t stream);

/*
 * sikv_sparse_attn -- fused dequantization + sparse attention
 * [SIKV 2.1.3, 2.1.4].
 *
 * For every query head (b, h*G+g), over the token set
 * T = [0, min(S, N_b)) U idx[b][h][0..k_b):
 *   logit_t = scale * q . K[t]                 for a sink (stored key),
 *   logit_t = scale * q . (mu + c[code(t)])    for a selected token;
 *   out     = sum_t softmax(logit)_t * V[t]    (fp32 accumulation).
 * Entries of idx are attended as listed (order does not matter; duplicates
 * count twice); an entry outside [S, N_b) sets SIKV_DEVERR_INDEX and is
 * skipped.  With an empty T the output row is 0.
 */
SIKV_API sikv_status sikv_sparse_attn(const sikv_params *p, const void *q, const void *K, const void *V,
                             const uint8_t *codes, const float *codebook, const float *mu,
                             const int32_t *idx, const int32_t *k_per_seq,
                             const int32_t *seq_lens, void *out, void *workspace,
                             size_t workspace_bytes, sikv_stream_t stream);

/*
 * sikv_append_codes -- decode-time append [SIKV 2.1.1, 2.1.3]: the code rows
 * of tokens [start[b], start[b] + count[b]) of every KV head of sequence b
 * become the sign codes of those tokens' keys (already written into K by the
 * caller) against the frozen prefill mean mu; all other rows, mu and the
 * codebook are left unchanged.  The pages describe prefill encoding only;
 * coding later keys against the frozen statistics is the plainest reading.
 *  - K: device [B][Hkv][Nmax][D]; mu: device fp32 [B][Hkv][D]; codes: device
 *    u8 [B][Hkv][Nmax][D/8], written in place.
 *  - start, count: device int32 [B]; a sequence with start < 0, count < 0 or
 *    start + count > Nmax sets SIKV_DEVERR_APPEND and is skipped.  The caller
 *    raises seq_lens afterwards to make the new tokens visible to decode.
 *  - workspace: sikv_append_workspace_size() bytes (the status header only).
 */
SIKV_API sikv_status sikv_append_codes(const sikv_params *p, const void *K, const int32_t *start,
                                       const int32_t *count, const float *mu, uint8_t *codes, void *workspace,
                                       size_t workspace_bytes, sikv_stream_t stream);

/*
 * sikv_decode -- one whole decode step: sikv_score, sikv_topk and
 * sikv_sparse_attn on the same inputs [SIKV 2.1.2-2.1.4].
 *
 * idx_out (may be NULL) receives the selected set as sikv_topk writes it;
 * scores_out (may be NULL) receives the scores as sikv_score writes them.
 */
SIKV_API sikv_status sikv_decode(const sikv_params *p, const void *q, const void *K, const void *V,
                        const uint8_t *codes, const float *codebook, const float *mu,
                        const int32_t *seq_lens, const int32_t *k_per_seq, void *out,
                        int32_t *idx_out, float *scores_out, void *workspace,
                        size_t workspace_bytes, sikv_stream_t stream);

/*
 * sikv_decode_host -- sikv_decode with the query and the output in host
 * memory: q_host and out_host are [B][Hq][D] in the cache dtype.  The query
 * is staged in the workspace: from a page-locked buffer (cudaHostAlloc,
 * cudaHostRegister; device-addressable) by a copy kernel that reads it once
 * over the host link, otherwise by cudaMemcpyAsync.  A page-locked output
 * buffer is written in place by the decode kernels; a pageable one is staged
 * through the workspace (pageable copies synchronize with the host).  Everything is
 * enqueued on `stream`; returns once enqueued, and out_host is valid after
 * the stream is synchronized.  K,
 * V, codes, codebook, mu, seq_lens and k_per_seq are device pointers as for
 * sikv_decode.  The workspace is sikv_decode_host_workspace_size() bytes:
 * the decode workspace followed by device copies of q and of the output.
 * Null host pointers return SIKV_ERR_INVALID_ARG; a failed copy returns
 * SIKV_ERR_CUDA.  The paper has no counterpart: this is the host-facing form
 * of the decode step [SIKV 2.1.2-2.1.4], one call per step for a caller
 * that keeps queries and outputs on the host.
 */
SIKV_API sikv_status sikv_decode_host(const sikv_params *p, const void *q_host, const void *K, const void *V,
                                      const uint8_t *codes, const float *codebook, const float *mu,
                                      const int32_t *seq_lens, const int32_t *k_per_seq, void *out_host,
                                      void *workspace, size_t workspace_bytes, sikv_stream_t stream);

/*
 * sikv_decode_host_plan -- sikv_decode_host for a serving loop that decodes
 * the same cache step after step: create() captures once, on the current
 * device, a CUDA graph of the step (a kernel that copies the query from
 * page-locked host memory into the workspace, the decode kernels, a kernel
 * that copies the output to page-locked host memory); run() points the two
 * copies at this step's buffers and launches the graph on `stream`, which
 * removes the gaps between separately launched kernels.  Same result bytes
 * as sikv_decode_host.
 *  - create: arguments as for sikv_decode_host (all device pointers and the
 *    workspace, sikv_decode_host_workspace_size() bytes, zeroed once by
 *    sikv_workspace_init; the plan keeps using it, so calls that share it --
 *    this plan's runs, other plans, other entry points -- must not overlap
 *    on the device).  *plan receives the handle.  Returns the
 *    argument errors of sikv_decode_host, SIKV_ERR_INVALID_ARG for a null
 *    plan pointer, SIKV_ERR_CUDA when the capture fails.
 *  - run: q_host and out_host are [B][Hq][D] in the cache dtype.  Page-locked
 *    buffers aligned to 16 bytes take the graph; others take
 *    sikv_decode_host's staged path on the same workspace.  Returns once
 *    enqueued; out_host is valid after `stream` is synchronized.  A plan is
 *    not thread-safe.
 *  - destroy: frees the graph (the workspace stays the caller's); NULL is a
 *    no-op.  Call it after the plan's work has finished.
 * The plan is a caller-owned host object; the executable graph's resources
 * are the CUDA runtime's, held from create to destroy (the library itself
 * still allocates no device memory).
 * The paper has no counterpart: this is the host-facing form of the decode
 * step [SIKV 2.1.2-2.1.4].
 */
typedef struct sikv_host_plan sikv_host_plan;
SIKV_API sikv_status sikv_decode_host_plan_create(const sikv_params *p, const void *K, const void *V,
                                                  const uint8_t *codes, const float *codebook, const float *mu,
                                                  const int32_t *seq_lens, const int32_t *k_per_seq, void *workspace,
                                                  size_t workspace_bytes, sikv_host_plan **plan);
SIKV_API sikv_status sikv_decode_host_plan_run(sikv_host_plan *plan, const void *q_host, void *out_host,
                                               sikv_stream_t stream);
SIKV_API void sikv_decode_host_plan_destroy(sikv_host_plan *plan);

/*
 * Comparison baselines -- not the method.  The pages compare the compressed-
 * domain retrieval with full dot-product scoring [SIKV 2.1.2] and the sparse
 * attention with dense attention [SIKV 2.1.4], and quote the speed-ups of
 * both in their efficiency results [SIKV 4]; these are the library's own
 * dense kernels for that comparison on the same GPU.  Layouts and errors as
 * above.
 *
 * sikv_dense_score: scores[b][h][t] = q_bar . K[b][h][t] (q_bar the sum of the
 * group's query heads, fp32 accumulation) for t in [S, N_b), -inf for sinks;
 * entries t >= N_b are not written.  workspace: the status header (256 B).
 *
 * sikv_dense_attn: out[b][hq] = softmax over every token t < N_b of
 * scale * q . K[t], applied to V, fp32 accumulation, written in the dtype.
 * workspace: sikv_dense_attn_workspace_size() bytes (split partials).
 */
SIKV_API sikv_status sikv_dense_score(const sikv_params *p, const void *q, const void *K, const int32_t *seq_lens,
                                      float *scores, void *workspace, size_t workspace_bytes, sikv_stream_t stream);
SIKV_API sikv_status sikv_dense_attn(const sikv_params *p, const void *q, const void *K, const void *V,
                                     const int32_t *seq_lens, void *out, void *workspace, size_t workspace_bytes,
                                     sikv_stream_t stream);

/*
 * 2-bit values -- the operating point the pages report accuracy for with
 * 2-bit quantization and a memory saving equal to 2-bit KIVI's [SIKV 3, 4];
 * the scheme is not given there.  This is KIVI's per-token value
 * quantization, read as:
 *   each token's row of V is cut into 4 groups of 32 channels; a group keeps
 *   m16 = fp16(min) and s16 = fp16(fl32(fl32(max - min) / 3)) (round to
 *   nearest even), and each value the level
 *       q = clamp(rint(fl32(fl32(v - m16) / s16)), 0, 3)   (ties to even; 0 when s16 = 0)
 *   that reads back as m16 + q * s16.  Values must lie in the fp16 range.
 * Row layout (48 bytes, the vq arrays below): 32 bytes of levels, dimension d
 * in bits 2 (d mod 4) of byte d / 4 (LSB first), then (m16, s16) of groups
 * 0..3, little-endian.  vq is device u8 [B][Hkv][Nmax][48], 16-byte aligned.
 *
 * sikv_quantize_values: rows t in [0, N_b) of vq from V (dtype
 * [B][Hkv][Nmax][D]); other rows are not written.  An invalid seq_lens[b]
 * sets SIKV_DEVERR_SEQ_LEN and skips the sequence.  workspace:
 * sikv_quantize_values_workspace_size() bytes (the status header).
 *
 * sikv_decode_qv / sikv_sparse_attn_qv: sikv_decode / sikv_sparse_attn with
 * the selected tokens' values read from vq; the sinks keep reading their
 * full-precision rows of V.  Arguments, workspaces and errors as there.
 */
SIKV_API sikv_status sikv_quantize_values(const sikv_params *p, const void *V, const int32_t *seq_lens, uint8_t *vq,
                                          void *workspace, size_t workspace_bytes, sikv_stream_t stream);
SIKV_API sikv_status sikv_decode_qv(const sikv_params *p, const void *q, const void *K, const void *V,
                                    const uint8_t *vq, const uint8_t *codes, const float *codebook, const float *mu,
                                    const int32_t *seq_lens, const int32_t *k_per_seq, void *out, int32_t *idx_out,
                                    float *scores_out, void *workspace, size_t workspace_bytes, sikv_stream_t stream);
SIKV_API sikv_status sikv_sparse_attn_qv(const sikv_params *p, const void *q, const void *K, const void *V,
                                         const uint8_t *vq, const uint8_t *codes, const float *codebook,
                                         const float *mu, const int32_t *idx, const int32_t *k_per_seq,
                                         const int32_t *seq_lens, void *out, void *workspace, size_t workspace_bytes,
                                         sikv_stream_t stream);

/*
 * sikv_kmeans_codebook -- comparison baseline, not the method: the iterative
 * K-means clustering that the one-pass sign-pattern codebook replaces
 * [SIKV 2.1.1], timed against it with 20 iterations [SIKV 4].  The pages
 * give no K-means details; this is Lloyd's algorithm on the same points and
 * codebook shape, for every (b, h):
 *   points  x[t][s] = fl32(K[t][4s:4s+4] - mu[4s:4s+4]) for t in [S, N_b);
 *   start   c[s][j] = x[init_idx[b][h][j]][s] for j < 16;
 *   iters   times: assign every point to the nearest centroid, minimizing
 *           ((d0*d0 + d1*d1) + d2*d2) + d3*d3 with d_i = x_i - c_i, each
 *           operation rounded to fp32 in that order, ties to the lower j;
 *           then move each non-empty cluster to the exact mean of its points
 *           rounded once to fp32 (an empty cluster keeps its centroid).
 * Outputs, in the layouts of sikv_encode_keys so that sikv_score reads them:
 *  - codes: device u8 [B][Hkv][Nmax][D/8]; rows t in [S, N_b) receive the
 *    last assignment, two codes per byte, even subspace in the low nibble;
 *    other rows are not written.
 *  - codebook: device fp32 [B][Hkv][D/4][16][4], the final centroids; it also
 *    holds the centroids between iterations.
 *  - counts: device int32 [B][Hkv][D/4][16], the last cluster sizes (may be NULL).
 * Inputs: K (dtype) [B][Hkv][Nmax][D], seq_lens [B], mu fp32 [B][Hkv][D] (the
 * channel mean of sikv_encode_keys), init_idx int32 [B][Hkv][16] (distinct
 * tokens in [S, N_b), drawn by the caller).  1 <= iters <= 1000, else
 * SIKV_ERR_INVALID_ARG.  Errors: an invalid seq_lens[b] sets
 * SIKV_DEVERR_SEQ_LEN and a start token outside [S, N_b) sets
 * SIKV_DEVERR_INDEX (its centroids start at 0); a sequence with N_b <= S
 * gets centroids 0 and counts 0.  The sums are exact while a cluster's
 * points span fewer than about 40 binades.
 *  - workspace: sikv_kmeans_workspace_size() bytes (chunk partials), on the
 *    device that runs the call.
 */
SIKV_API sikv_status sikv_kmeans_codebook(const sikv_params *p, const void *K, const int32_t *seq_lens,
                                          const float *mu, const int32_t *init_idx, int32_t iters, uint8_t *codes,
                                          float *codebook, int32_t *counts, void *workspace, size_t workspace_bytes,
                                          sikv_stream_t stream);

/*
 * sikv_sparse_attn_static -- sikv_sparse_attn for callers that cannot
 * allocate device memory.  The paper has no counterpart: it is a deployment
 * variant of the attention step.
 *
 * Some callers cannot call cudaMalloc, so they cannot hand the library a
 * workspace: a serving engine that carves up device memory once at start-up
 * and may not allocate inside its decode loop, or a plugin host that passes a
 * kernel only its input and output buffers.  This call computes exactly what
 * sikv_sparse_attn computes, with the same arguments minus the workspace; its
 * scratch (split-k partials and the device status word) lives in an 8 MiB
 * array compiled into the library, which every GPU that loads the library
 * holds until the process exits.
 *  - Limit: the partials, B * Hkv * ceil((S + kmax) / 128) * G * 520 bytes
 *    plus 256, must fit in 8 MiB; larger sizes return SIKV_ERR_WORKSPACE and
 *    launch nothing.  Invalid parameters return SIKV_ERR_INVALID_ARG.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it for the life of the process; make
 *    that first call before any stream capture.  The cache does not survive
 *    cudaDeviceReset (or any teardown of the device's primary context): after
 *    one, the cached address is stale and this entry point must not be called
 *    again in that process.
 *  - All calls share the one array: calls that may overlap on the GPU (on
 *    different streams, or from different threads) race and must be ordered
 *    by the caller.
 *  - device_flags (device int32, may be NULL) receives the SIKV_DEVERR_* bits
 *    of this call.  Nothing is allocated: no cudaMalloc, no cudaFree.
 */
SIKV_API sikv_status sikv_sparse_attn_static(const sikv_params *p, const void *q, const void *K,
                                             const void *V, const uint8_t *codes, const float *codebook,
                                             const float *mu, const int32_t *idx, const int32_t *k_per_seq,
                                             const int32_t *seq_lens, void *out, int32_t *device_flags,
                                             sikv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SIKV_H */
